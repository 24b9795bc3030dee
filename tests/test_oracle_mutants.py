"""Mutation check of the oracle's pins.

Each entry below plants one plausible mistake in the fp64 oracle, on the CPU
only: a dropped or mis-signed term, an off-by-one range, a transposed operand,
a wrong tie rule, a missing shift.  Every pin of ``test_oracle_pins.py`` is
run against the mutated oracle, and at least one of them must fail; a mistake
that no pin notices is a gap in the pins.  The mutants live here, in the test;
the oracle itself is never edited.
"""

import dataclasses
import math

import numpy as np
import pytest

import oracle as O
import oracle.hybrid as OH
import test_oracle_pins as P


# ----------------------------------------------------------------------------- the battery

def _battery():
    """Every pin test with every parameter set, as (name, callable)."""
    out = []
    for name in sorted(dir(P)):
        fn = getattr(P, name)
        if not (name.startswith("test_") and callable(fn)):
            continue
        sets = [{}]
        for mark in getattr(fn, "pytestmark", []):
            if mark.name != "parametrize":
                continue
            names = [s.strip() for s in mark.args[0].split(",")]
            values = [v if len(names) > 1 else (v,) for v in mark.args[1]]
            sets = [dict(base, **dict(zip(names, v))) for base in sets for v in values]
        for kw in sets:
            out.append((f"{name}{sorted(kw.items()) if kw else ''}", lambda fn=fn, kw=kw: fn(**kw)))
    return out


def _failing_pins():
    failed = []
    for name, run in _battery():
        try:
            run()
        except Exception:  # an assertion, or a crash the mistake causes
            failed.append(name)
    return failed


# ----------------------------------------------------------------------------- mutants

def _partition_oldest_partial(orig):
    def f(T, S, W, Bk):  # blocks aligned to the window side: the partial block is the oldest
        p = orig(T, S, W, Bk)
        a, b = p.evicted
        blocks = []
        while b > a:
            blocks.append((max(a, b - Bk), b))
            b -= Bk
        return dataclasses.replace(p, blocks=tuple(reversed(blocks)))
    return f


def _partition_drop_ragged(orig):
    def f(T, S, W, Bk):
        p = orig(T, S, W, Bk)
        if p.blocks and p.blocks[-1][1] - p.blocks[-1][0] < Bk:
            return dataclasses.replace(p, blocks=p.blocks[:-1])
        return p
    return f


def _state_with_window(orig):
    def f(K, V, part):
        if part.T > part.evicted[0]:
            part = dataclasses.replace(part, evicted=(part.evicted[0], part.T))
        return orig(K, V, part)
    return f


def _stats_sample_variance(orig):
    def f(K, part):
        mu, var = orig(K, part)
        for j, (a, b) in enumerate(part.blocks):
            if b - a > 1:
                var[j] = var[j] * (b - a) / (b - a - 1)
        return mu, var
    return f


def _scores(c2=0.5, second_sign=1.0, square="qs", heads="sum", spread="var"):
    """The block score with one knob turned (defaults: the oracle's reading)."""
    def f(q, mu, var, scale):
        q = np.asarray(q, dtype=np.float64)
        qs = q * scale
        sq = qs * qs if square == "qs" else qs * q
        v = var if spread == "var" else np.sqrt(var)
        s = qs @ mu.T + second_sign * c2 * (sq @ v.T)
        return s.sum(axis=0) if heads == "sum" else s.mean(axis=0)
    return lambda orig: f


def _select(tie="low", k_off=0, order="asc"):
    def f(scores, k):
        nb = scores.shape[0]
        key = (lambda j: (-scores[j], j)) if tie == "low" else (lambda j: (-scores[j], -j))
        top = sorted(range(nb), key=key)[: max(0, min(k + k_off, nb))]
        return np.array(sorted(top) if order == "asc" else top, dtype=np.int64)
    return lambda orig: f


def _strided_first_of_group(orig):
    return lambda nb, stride: np.array([j for j in range(nb) if j % stride == 0], dtype=np.int64)


def _strided_topk_over_all(orig):
    def f(scores, k, stride):  # the top-k taken over every block, strided ones included
        nb = scores.shape[0]
        fixed = set(int(j) for j in OH.strided_blocks(nb, stride))
        top = sorted(range(nb), key=lambda j: (-scores[j], j))[: min(k, nb)]
        return np.array(sorted(fixed | set(top)), dtype=np.int64)
    return f


def _mask_without_sinks(orig):
    def f(part, sel):
        m = orig(part, sel)
        m[part.sink[0]:part.sink[1]] = False
        w0, w1 = part.window
        m[w0:w1] = True
        return m
    return f


def _direct(lin_kernel="taylor", lin_shift=True):
    def f(q, K, V, part, sel, scale):
        T = part.T
        s = (np.asarray(q, dtype=np.float64) * scale) @ np.asarray(K[:T], dtype=np.float64).T
        X = OH.exact_mask(part, sel)
        L = np.zeros(T, dtype=bool)
        L[part.evicted[0]:part.evicted[1]] = True
        lin = L & ~X
        m = s[:, X].max(axis=1, keepdims=True) if X.any() else np.zeros((s.shape[0], 1))
        wx = np.where(X[None, :], np.exp(s - m), 0.0)
        lw = (1.0 + s) if lin_kernel == "taylor" else np.exp(s)
        wl = np.where(lin[None, :], lw * (np.exp(-m) if lin_shift else 1.0), 0.0)
        w = wx + wl
        return (w @ np.asarray(V[:T], dtype=np.float64)) / w.sum(axis=1, keepdims=True)
    return lambda orig: f


def _subtract(one=1.0, sign=-1.0, shift=True, h_t=False):
    """The subtraction form with one knob turned (defaults: the oracle's)."""
    def f(q, K, V, part, sel, scale, state=None):
        qs = np.asarray(q, dtype=np.float64) * scale
        H, zk, zv, n = state if state is not None else OH.linear_state(K, V, part)
        if h_t:
            H = H.T
        idx = np.nonzero(OH.exact_mask(part, sel))[0]
        Kx, Vx = np.asarray(K[idx], dtype=np.float64), np.asarray(V[idx], dtype=np.float64)
        s_x = qs @ Kx.T
        m = s_x.max(axis=1, keepdims=True) if idx.size else np.zeros((qs.shape[0], 1))
        p = np.exp(s_x - m)
        sel_tok = np.zeros(part.T, dtype=bool)
        for j in sel:
            a, b = part.blocks[int(j)]
            sel_tok[a:b] = True
        sidx = np.nonzero(sel_tok)[0]
        Ks, Vs = np.asarray(K[sidx], dtype=np.float64), np.asarray(V[sidx], dtype=np.float64)
        w_sel = one + qs @ Ks.T
        em = np.exp(-m) if shift else np.ones_like(m)
        num = p @ Vx + em * (zv[None, :] + qs @ H + sign * (w_sel @ Vs))
        den = p.sum(axis=1, keepdims=True) + em * (n + qs @ zk + sign * w_sel.sum(axis=1))[:, None]
        return num / den
    return lambda orig: f


def _softmax_unscaled(orig):
    return lambda q, K, V, T, scale: orig(q, K, V, T, 1.0)


def _taylor_as_exp(orig):
    return lambda q, K, V, T, scale: OH.full_softmax(q, K, V, T, scale)


def _brute_window_short(orig):
    return lambda q, K, V, T, S, W, Bk, sel, scale: orig(q, K, V, T, S, max(W - 1, 0), Bk, sel, scale)


def _append_wrong_token(orig):
    def f(self, k, v):  # folds the token at T - W (one too new) instead of T - 1 - W
        k = np.asarray(k, dtype=np.float64)
        v = np.asarray(v, dtype=np.float64)
        if self.T >= self.K.shape[0]:
            grow = max(16, self.K.shape[0])
            self.K = np.vstack([self.K, np.zeros((grow, self.K.shape[1]))])
            self.V = np.vstack([self.V, np.zeros((grow, self.V.shape[1]))])
        self.K[self.T] = k
        self.V[self.T] = v
        self.T += 1
        p = self.T - self.W
        if self.S <= p < self.T:
            kp, vp = self.K[p], self.V[p]
            self.H = self.H + np.outer(kp, vp)
            self.zk = self.zk + kp
            self.zv = self.zv + vp
            self.n += 1.0
            j = (p - self.S) // self.Bk
            while j >= len(self.bsum):
                self.bsum.append(np.zeros_like(kp))
                self.bsq.append(np.zeros_like(kp))
                self.bcnt.append(0)
            self.bsum[j] = self.bsum[j] + kp
            self.bsq[j] = self.bsq[j] + kp * kp
            self.bcnt[j] += 1
    return f


def _unit_stats_uncentred(orig):
    def f(self):
        mu, var = orig(self)
        return mu, var + mu * mu
    return f


# (what is replaced, how) -> the planted mistake
MUTANTS = {
    "partition: window one token wider": ("partition", lambda o: lambda T, S, W, Bk: o(T, S, W + 1, Bk)),
    "partition: one sink too few": ("partition", lambda o: lambda T, S, W, Bk: o(T, max(S - 1, 0), W, Bk)),
    "partition: the partial block is the oldest": ("partition", _partition_oldest_partial),
    "partition: the ragged newest block is dropped": ("partition", _partition_drop_ragged),
    "linear_state: H transposed": ("linear_state", lambda o: lambda K, V, p: (lambda r: (r[0].T,) + r[1:])(o(K, V, p))),
    "linear_state: zk and zv swapped": ("linear_state", lambda o: lambda K, V, p: (lambda r: (r[0], r[2], r[1], r[3]))(o(K, V, p))),
    "linear_state: n off by one": ("linear_state", lambda o: lambda K, V, p: (lambda r: r[:3] + (r[3] + 1.0,))(o(K, V, p))),
    "linear_state: the window folded in too": ("linear_state", _state_with_window),
    "block_stats: sample variance": ("block_stats", _stats_sample_variance),
    "block_stats: uncentred second moment": ("block_stats", lambda o: lambda K, p: (lambda r: (r[0], r[1] + r[0] ** 2))(o(K, p))),
    "block_scores: the 1/2 dropped": ("block_scores", _scores(c2=1.0)),
    "block_scores: second-order term subtracted": ("block_scores", _scores(second_sign=-1.0)),
    "block_scores: scale not squared in the second-order term": ("block_scores", _scores(square="q")),
    "block_scores: mean over the group's heads": ("block_scores", _scores(heads="mean")),
    "block_scores: standard deviation for variance": ("block_scores", _scores(spread="std")),
    "select_blocks: ties to the higher index": ("select_blocks", _select(tie="high")),
    "select_blocks: one block too few": ("select_blocks", _select(k_off=-1)),
    "select_blocks: returned in score order": ("select_blocks", _select(order="score")),
    "strided_blocks: first block of each group": ("strided_blocks", _strided_first_of_group),
    "select_blocks_strided: top-k over every block": ("select_blocks_strided", _strided_topk_over_all),
    "exact_mask: sinks left out": ("exact_mask", _mask_without_sinks),
    "hybrid_direct: exact kernel for linear tokens": ("hybrid_direct", _direct(lin_kernel="exp")),
    "hybrid_direct: linear weights not shifted by the max": ("hybrid_direct", _direct(lin_shift=False)),
    "hybrid_subtract: the 1 of 1 + s dropped for the selected blocks": ("hybrid_subtract", _subtract(one=0.0)),
    "hybrid_subtract: selected blocks added, not subtracted": ("hybrid_subtract", _subtract(sign=1.0)),
    "hybrid_subtract: linear part not shifted by the max": ("hybrid_subtract", _subtract(shift=False)),
    "hybrid_subtract: H read transposed": ("hybrid_subtract", _subtract(h_t=True)),
    "full_softmax: scale missing": ("full_softmax", _softmax_unscaled),
    "pure_taylor: exp(s) for 1 + s": ("pure_taylor", _taylor_as_exp),
    "brute_force_hybrid: window one token short": ("brute_force_hybrid", _brute_window_short),
    "OracleUnit.append: folds the token one too new": ("OracleUnit.append", _append_wrong_token),
    "OracleUnit.stats: uncentred second moment": ("OracleUnit.stats", _unit_stats_uncentred),
}


def _plant(monkeypatch, target, make):
    if target.startswith("OracleUnit."):
        attr = target.split(".", 1)[1]
        monkeypatch.setattr(OH.OracleUnit, attr, make(getattr(OH.OracleUnit, attr)))
        return
    mutant = make(getattr(OH, target))
    monkeypatch.setattr(OH, target, mutant)   # calls inside the oracle module
    monkeypatch.setattr(O, target, mutant)    # calls through the package, as the pins make them


def test_knob_defaults_are_the_oracle():
    """The re-typed variants above, with their knobs at the oracle's reading,
    agree with the oracle (so a mutant differs from it by its knob alone)."""
    rng = np.random.default_rng(5)
    T, S, W, Bk, d, G = 150, 3, 20, 8, 6, 2
    K, V = rng.standard_normal((T, d)), rng.standard_normal((T, d))
    q = rng.standard_normal((G, d))
    part = O.partition(T, S, W, Bk)
    mu, var = O.block_stats(K, part)
    scale = 1 / math.sqrt(d)
    np.testing.assert_allclose(_scores()(None)(q, mu, var, scale), O.block_scores(q, mu, var, scale), atol=1e-13)
    sc = O.block_scores(q, mu, var, scale)
    assert list(_select()(None)(sc, 5)) == list(O.select_blocks(sc, 5))
    sel = O.select_blocks(sc, 5)
    np.testing.assert_allclose(_direct()(None)(q, K, V, part, sel, scale), O.hybrid_direct(q, K, V, part, sel, scale),
                               atol=1e-13)
    np.testing.assert_allclose(_subtract()(None)(q, K, V, part, sel, scale),
                               O.hybrid_subtract(q, K, V, part, sel, scale), atol=1e-13)


def test_unmutated_oracle_passes_the_battery():
    assert _failing_pins() == []


@pytest.mark.filterwarnings("ignore::RuntimeWarning")  # a mutant may divide by a zero normaliser
@pytest.mark.parametrize("mistake", sorted(MUTANTS))
def test_a_pin_catches_the_planted_mistake(mistake, monkeypatch):
    target, make = MUTANTS[mistake]
    _plant(monkeypatch, target, make)
    assert _failing_pins(), f"no pin fails with the planted mistake: {mistake}"
