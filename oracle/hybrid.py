"""fp64 oracle: the decode-step hybrid attention written out plainly, in numpy.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  Everything is fp64; bf16
inputs are converted exactly.  One "unit" is one (layer, batch row, KV head): a
key/value history ``K, V`` of shape [T, d] and the ``G`` query heads of that KV
head's group, ``q`` of shape [G, d].

Sources (page title, then the part of the page):

* SALSA: Training-Consistent Sparse Caching with Sink Preservation for
  Linearized LLMs -- abstract: history is split into a sliding window, a sparse
  global cache and a linear-attention hidden state; initial sink tokens are kept
  with the window.
* SPLA: Block Sparse Plus Linear Attention for Long Context Modeling --
  Abstract and TL;DR: blocks for exact attention are picked by a metric from a
  second-order Taylor expansion around block statistics; unselected blocks go
  through residual linear attention (RLA), computed as global linear attention
  minus the selected blocks' linear attention, so unselected blocks are never
  read.  Table of contents: "Grouped Sparsity", "Principled Block Selection via
  Taylor Expansion", "Recurrence", "IO-Efficient Implementation".
* SLAKE: Softmax-Approximated Training-Free Linear Attention with KV-Cache
  Eviction for Long-Sequence LLMs -- Abstract (PTAA): a first-order Taylor
  expansion linearises the softmax kernel for low-importance tokens, while
  high-salience tokens keep the exact softmax kernel.

Readings where the pages are silent (the plainest reading the rest supports):

* R1 the linear state holds only evicted tokens [S, T-W) (neither sinks nor
  window); blocks tile that range from position S, the newest block may be
  partial and is a candidate;
* R2 block statistics are the mean and the population variance (divide by the
  count);
* R3 the score of block j for one query is q'.mu_j + 1/2 sum_c q'_c^2 var_jc with
  q' = q * scale, scale = 1/sqrt(d): the first two terms of the cumulant
  expansion of log E[exp(q'.k)] about the block mean;
* R4 one selection per KV head ("Grouped Sparsity"): the group score is the sum
  of its query heads' scores;
* R5 top-k by score, ties to the lower block index, output ascending; nb <= k
  selects every block;
* R6 the Taylor kernel is exp(s) ~ 1 + s with the same scaled s, no clamp;
* R7 one normaliser: exact weights exp(s_t), linear weights (1 + s_t), one sum in
  the denominator;
* R8 strided block selection (SPLA, table of contents: the section's heading
  only): a fixed stride of always-exact blocks -- the last block of every
  `stride` consecutive candidate blocks -- plus the top-k among the rest.  The
  page gives no definition, so this is one reading of the heading, not the
  page's method; it is pinned to its own definition only.

Pins (tests/test_oracle_pins.py): every function here is pinned by at least one
check that does not retype it -- all-selected equals full softmax, empty exact
set equals pure Taylor, subtraction form equals direct form, q = 0 gives the
mean of V, the score against the Gaussian moment generating function and a
cubic-remainder test, top-k against exhaustive search, the incremental state
against the direct definition, and the whole operator against a token-by-token
brute force on tiny inputs and a hand-derived closed form.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np


# ----------------------------------------------------------------------------- partition

@dataclasses.dataclass(frozen=True)
class Partition:
    """Split of positions [0, T) of one unit (SALSA abstract; SPLA abstract)."""
    T: int
    sink: tuple       # [0, min(S, T))
    window: tuple     # [max(S, T - W), T)  (empty when T <= S)
    evicted: tuple    # [S, T - W) when T > S + W, else empty   (R1)
    blocks: tuple     # block j = [S + j*Bk, min(S + (j+1)*Bk, T - W))

    @property
    def nb(self) -> int:
        return len(self.blocks)


def partition(T: int, S: int, W: int, Bk: int) -> Partition:
    sink = (0, min(S, T))
    if T > S:
        window = (max(S, T - W), T)
    else:
        window = (T, T)
    if T > S + W:
        ev = (S, T - W)
    else:
        ev = (S, S)
    blocks = []
    a = ev[0]
    while a < ev[1]:
        blocks.append((a, min(a + Bk, ev[1])))
        a += Bk
    return Partition(T, sink, window, ev, tuple(blocks))


# ----------------------------------------------------------------------------- state

def linear_state(K: np.ndarray, V: np.ndarray, part: Partition):
    """Global linear-attention state over the evicted tokens L (R1).

    H = sum_{t in L} k_t v_t^T  ([d, d], row index = key channel),
    zk = sum k_t, zv = sum v_t, n = |L|.  SPLA, "Residual Linear Attention (RLA)"
    with the first-order Taylor feature map of SLAKE (PTAA): 1 + q'.k expands to
    the pair (1, q') against (1, k).
    """
    a, b = part.evicted
    KL = np.asarray(K[a:b], dtype=np.float64)
    VL = np.asarray(V[a:b], dtype=np.float64)
    H = KL.T @ VL
    return H, KL.sum(axis=0), VL.sum(axis=0), float(b - a)


def block_stats(K: np.ndarray, part: Partition):
    """Per-block mean and population variance of the keys (R2).  [nb, d] each."""
    d = K.shape[1]
    mu = np.zeros((part.nb, d))
    var = np.zeros((part.nb, d))
    for j, (a, b) in enumerate(part.blocks):
        kb = np.asarray(K[a:b], dtype=np.float64)
        mu[j] = kb.mean(axis=0)
        var[j] = ((kb - mu[j]) ** 2).mean(axis=0)
    return mu, var


# ----------------------------------------------------------------------------- selection

def block_scores(q: np.ndarray, mu: np.ndarray, var: np.ndarray, scale: float) -> np.ndarray:
    """Group score of every candidate block (R3, R4).

    SPLA, "Principled Block Selection via Taylor Expansion": per query head i,
    q_i'.mu_j + 1/2 * q_i'^T diag(var_j) q_i', summed over the group's heads.
    """
    qs = np.asarray(q, dtype=np.float64) * scale            # [G, d]
    first = qs @ mu.T                                         # [G, nb]
    second = 0.5 * ((qs * qs) @ var.T)                        # [G, nb]
    return (first + second).sum(axis=0)


def select_blocks(scores: np.ndarray, k: int) -> np.ndarray:
    """Top-k block indices (R5): larger score first, ties to the lower index,
    returned in ascending index order."""
    nb = scores.shape[0]
    order = sorted(range(nb), key=lambda j: (-scores[j], j))
    return np.array(sorted(order[: min(k, nb)]), dtype=np.int64)


def strided_blocks(nb: int, stride: int) -> np.ndarray:
    """The always-exact blocks of strided block selection (R8): the last block
    of every group of `stride` consecutive candidate blocks, j % stride ==
    stride - 1 (none when stride > nb; every block when stride == 1)."""
    return np.array([j for j in range(nb) if j % stride == stride - 1], dtype=np.int64)


def select_blocks_strided(scores: np.ndarray, k: int, stride: int) -> np.ndarray:
    """Strided block selection (R8): the strided blocks, plus the top-k by
    score among the other blocks (larger score first, ties to the lower
    index); ascending."""
    nb = scores.shape[0]
    fixed = set(int(j) for j in strided_blocks(nb, stride))
    rest = [j for j in range(nb) if j not in fixed]
    order = sorted(rest, key=lambda j: (-scores[j], j))
    return np.array(sorted(fixed | set(order[: min(k, len(rest))])), dtype=np.int64)


def exact_mask(part: Partition, sel) -> np.ndarray:
    """Boolean mask over [0, T) of the exactly attended set X = sinks u window u
    selected blocks (SALSA abstract; SPLA abstract)."""
    m = np.zeros(part.T, dtype=bool)
    m[part.sink[0]:part.sink[1]] = True
    m[part.window[0]:part.window[1]] = True
    for j in sel:
        a, b = part.blocks[int(j)]
        m[a:b] = True
    return m


# ----------------------------------------------------------------------------- attention

def _scores(q, K, T, scale):
    return (np.asarray(q, dtype=np.float64) * scale) @ np.asarray(K[:T], dtype=np.float64).T


def hybrid_direct(q, K, V, part: Partition, sel, scale: float) -> np.ndarray:
    """Direct form: exact softmax weights exp(s_t) on X, Taylor weights (1 + s_t)
    on the evicted tokens outside the selected blocks, one shared normaliser
    (SLAKE abstract, PTAA; R6, R7).  Sums over L minus selected explicitly."""
    T = part.T
    s = _scores(q, K, T, scale)                               # [G, T]
    X = exact_mask(part, sel)
    L = np.zeros(T, dtype=bool)
    L[part.evicted[0]:part.evicted[1]] = True
    lin = L & ~X
    m = s[:, X].max(axis=1, keepdims=True) if X.any() else np.zeros((s.shape[0], 1))
    wx = np.where(X[None, :], np.exp(s - m), 0.0)
    wl = np.where(lin[None, :], (1.0 + s) * np.exp(-m), 0.0)
    w = wx + wl
    Vt = np.asarray(V[:T], dtype=np.float64)
    return (w @ Vt) / w.sum(axis=1, keepdims=True)


def hybrid_subtract(q, K, V, part: Partition, sel, scale: float, state=None) -> np.ndarray:
    """Subtraction form (SPLA abstract; "IO-Efficient Implementation"): the
    residual linear term is the global state's term minus the selected blocks'
    own Taylor terms, so no unselected token is touched.

    o = (N_ex + e^{-m} (N_glob - N_sel)) / (D_ex + e^{-m} (D_glob - D_sel))
    with N_glob = zv + H^T q', D_glob = n + q'.zk.
    """
    G = q.shape[0]
    qs = np.asarray(q, dtype=np.float64) * scale
    if state is None:
        state = linear_state(K, V, part)
    H, zk, zv, n = state
    X = exact_mask(part, sel)
    idx = np.nonzero(X)[0]
    Kx = np.asarray(K[idx], dtype=np.float64)
    Vx = np.asarray(V[idx], dtype=np.float64)
    s_x = qs @ Kx.T                                           # [G, |X|]
    m = s_x.max(axis=1, keepdims=True) if idx.size else np.zeros((G, 1))
    p = np.exp(s_x - m)
    N_ex = p @ Vx
    D_ex = p.sum(axis=1, keepdims=True)
    N_glob = zv[None, :] + qs @ H
    D_glob = n + qs @ zk
    sel_tok = np.zeros(part.T, dtype=bool)
    for j in sel:
        a, b = part.blocks[int(j)]
        sel_tok[a:b] = True
    sidx = np.nonzero(sel_tok)[0]
    Ks = np.asarray(K[sidx], dtype=np.float64)
    Vs = np.asarray(V[sidx], dtype=np.float64)
    w_sel = 1.0 + qs @ Ks.T                                   # [G, |sel tokens|]
    N_sel = w_sel @ Vs
    D_sel = w_sel.sum(axis=1)
    em = np.exp(-m)
    num = N_ex + em * (N_glob - N_sel)
    den = D_ex + em * (D_glob - D_sel)[:, None]
    return num / den


def full_softmax(q, K, V, T: int, scale: float) -> np.ndarray:
    """Plain softmax attention over [0, T)."""
    s = _scores(q, K, T, scale)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    return (p @ np.asarray(V[:T], dtype=np.float64)) / p.sum(axis=1, keepdims=True)


def pure_taylor(q, K, V, T: int, scale: float) -> np.ndarray:
    """First-order Taylor (exp(s) ~ 1 + s) attention over [0, T) (SLAKE, PTAA)."""
    w = 1.0 + _scores(q, K, T, scale)
    return (w @ np.asarray(V[:T], dtype=np.float64)) / w.sum(axis=1, keepdims=True)


def brute_force_hybrid(q, K, V, T, S, W, Bk, sel, scale) -> np.ndarray:
    """Token-by-token definition with Python loops (tiny inputs only): classify
    each position, weight it exp(s) or (1 + s), normalise once."""
    G, d = q.shape
    out = np.zeros((G, d))
    chosen = set(int(j) for j in sel)
    for i in range(G):
        num = [0.0] * d
        den = 0.0
        for t in range(T):
            s = 0.0
            for c in range(d):
                s += float(q[i, c]) * scale * float(K[t, c])
            if t < S or t >= T - W:
                w = math.exp(s)                      # sink or window
            else:
                j = (t - S) // Bk                    # evicted: block j
                w = math.exp(s) if j in chosen else 1.0 + s
            den += w
            for c in range(d):
                num[c] += w * float(V[t, c])
        out[i] = np.array(num) / den
    return out


# ----------------------------------------------------------------------------- stateful unit

class OracleUnit:
    """One unit with its own incremental append (the RLA recurrence, SPLA
    "Recurrence"), in fp64.  Keys and values are stored; the linear state and the
    block statistics are maintained by rank-1 / running-sum updates, not
    recomputed, so that comparing them with ``linear_state``/``block_stats``
    checks the recurrence."""

    def __init__(self, K0, V0, S: int, W: int, Bk: int, k: int, scale: float, capacity=None):
        K0 = np.asarray(K0, dtype=np.float64)
        V0 = np.asarray(V0, dtype=np.float64)
        T0, d = K0.shape
        cap = capacity or T0
        self.K = np.zeros((cap, d))
        self.V = np.zeros((cap, d))
        self.K[:T0] = K0
        self.V[:T0] = V0
        self.S, self.W, self.Bk, self.k, self.scale = S, W, Bk, k, scale
        self.T = T0
        part = partition(T0, S, W, Bk)
        self.H, self.zk, self.zv, self.n = linear_state(self.K, self.V, part)
        self.bsum = [np.asarray(self.K[a:b]).sum(axis=0) for (a, b) in part.blocks]
        self.bsq = [(np.asarray(self.K[a:b]) ** 2).sum(axis=0) for (a, b) in part.blocks]
        self.bcnt = [b - a for (a, b) in part.blocks]

    @property
    def part(self) -> Partition:
        return partition(self.T, self.S, self.W, self.Bk)

    def append(self, k, v):
        """Write token T; the token leaving the window (position T - W after the
        write, if it is past the sinks) is folded into H, zk, zv, n and into the
        running sums of its block."""
        k = np.asarray(k, dtype=np.float64)
        v = np.asarray(v, dtype=np.float64)
        if self.T >= self.K.shape[0]:
            grow = max(16, self.K.shape[0])
            self.K = np.vstack([self.K, np.zeros((grow, self.K.shape[1]))])
            self.V = np.vstack([self.V, np.zeros((grow, self.V.shape[1]))])
        self.K[self.T] = k
        self.V[self.T] = v
        self.T += 1
        p = self.T - 1 - self.W
        if p >= self.S:
            kp, vp = self.K[p], self.V[p]
            self.H = self.H + np.outer(kp, vp)
            self.zk = self.zk + kp
            self.zv = self.zv + vp
            self.n += 1.0
            j = (p - self.S) // self.Bk
            if j == len(self.bsum):
                self.bsum.append(np.zeros_like(kp))
                self.bsq.append(np.zeros_like(kp))
                self.bcnt.append(0)
            self.bsum[j] = self.bsum[j] + kp
            self.bsq[j] = self.bsq[j] + kp * kp
            self.bcnt[j] += 1

    def stats(self):
        """Block mean and population variance from the running sums."""
        if not self.bcnt:
            d = self.K.shape[1]
            return np.zeros((0, d)), np.zeros((0, d))
        c = np.array(self.bcnt, dtype=np.float64)[:, None]
        mu = np.array(self.bsum) / c
        var = np.array(self.bsq) / c - mu * mu
        return mu, np.maximum(var, 0.0)

    def state(self):
        return self.H, self.zk, self.zv, self.n

    def decode(self, q, sel=None):
        """One decode step for the group's queries ``q`` [G, d]: returns
        (out [G, d], selection, scores).  With ``sel`` given, that selection is
        used instead of the top-k (the scores are still returned)."""
        part = self.part
        mu, var = self.stats()
        scores = block_scores(q, mu, var, self.scale) if part.nb else np.zeros(0)
        if sel is None:
            sel = select_blocks(scores, self.k)
        out = hybrid_subtract(q, self.K, self.V, part, sel, self.scale, state=self.state())
        return out, np.asarray(sel, dtype=np.int64), scores
