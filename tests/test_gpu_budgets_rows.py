"""Per-KV-head budgets (each KV head its own window and top-k) and per-row
lengths (each batch row its own history length), through the C ABI against the
fp64 oracle unit by unit: every unit is the plain method at its own (T_b, W_h,
k_h).  Covers decodes, fused decode + append steps, chunked appends (the dense
fold of each unit's own evictions), state sync and checkpoint restore."""

import math

import numpy as np
import pytest

import oracle as O
from harness import OUT_MAX_ABS, OUT_REL_L2, SEL_TIE, STATE_REL, bf16_bits, bits_to_f64, check_outputs, \
    check_selection, to_device_bf16

pytestmark = pytest.mark.gpu


class RaggedCase:
    """A layer whose rows have lengths row_T0[b] and whose KV heads have
    budgets (head_W[h], head_k[h]); n_app tokens per row can be appended."""

    def __init__(self, B, Hq, Hkv, d, row_T0, Bk, S, head_W, head_k, n_app=0, seed=0):
        import torch
        from hybrid_sparse_linear_decode_b200 import HybridAttentionLayer, make_config
        self.B, self.Hq, self.Hkv, self.d, self.G = B, Hq, Hkv, d, Hq // Hkv
        self.S, self.Bk = S, Bk
        self.W, self.k = list(head_W), list(head_k)
        self.T = list(row_T0)
        self.scale = 1 / math.sqrt(d)
        self.rng = np.random.default_rng(seed)
        cap = max(row_T0) + n_app
        self.Kb = bf16_bits(self.rng.standard_normal((B, Hkv, cap, d)))
        self.Vb = bf16_bits(self.rng.standard_normal((B, Hkv, cap, d)))
        self.K, self.V = bits_to_f64(self.Kb), bits_to_f64(self.Vb)
        uniform = len(set(self.W)) == 1 and len(set(self.k)) == 1
        self.cfg = make_config(B, Hq, Hkv, d, Bk, S, min(self.W), max(self.k), cap,
                               head_window=None if uniform else self.W, head_top_k=None if uniform else self.k)
        self.layer = HybridAttentionLayer(self.cfg, "cuda")
        dev = self.layer.device
        for b in range(B):
            t = row_T0[b]
            self.layer.k_cache[b, :, :t].copy_(to_device_bf16(self.Kb[b, :, :t], dev))
            self.layer.v_cache[b, :, :t].copy_(to_device_bf16(self.Vb[b, :, :t], dev))
        self.layer.init(list(row_T0) if len(set(row_T0)) > 1 else int(row_T0[0]))
        torch.cuda.synchronize()
        assert self.layer.row_lengths() == self.T

    def kmax(self):
        return max(self.k)

    def new_tokens(self, n=1):
        """bf16 bits of each row's next n tokens: [B][Hkv][n][d] (row b's token i at T_b + i)."""
        kb = np.stack([self.Kb[b, :, self.T[b]:self.T[b] + n] for b in range(self.B)])
        vb = np.stack([self.Vb[b, :, self.T[b]:self.T[b] + n] for b in range(self.B)])
        return kb, vb

    def oracle_unit(self, qb, b, h, sel=None):
        T = self.T[b]
        K, V = self.K[b, h, :T], self.V[b, h, :T]
        part = O.partition(T, self.S, self.W[h], self.Bk)
        q = bits_to_f64(qb)[b, h * self.G:(h + 1) * self.G]
        mu, var = O.block_stats(K, part)
        scores = O.block_scores(q, mu, var, self.scale) if part.nb else np.zeros(0)
        use = O.select_blocks(scores, self.k[h]) if sel is None else sel
        return O.hybrid_subtract(q, K, V, part, use, self.scale), scores

    def check_decode(self, qb, out, sel):
        refs, gots = [], []
        for b in range(self.B):
            for h in range(self.Hkv):
                _, scores = self.oracle_unit(qb, b, h)
                row = sel[b, h]
                kh = self.k[h]
                assert all(j == -1 for j in row[kh:]), row     # past the head's own top-k
                check_selection(row[:kh], scores, kh)
                gsel = np.array([int(j) for j in row if j >= 0], dtype=np.int64)
                ref, _ = self.oracle_unit(qb, b, h, sel=gsel)
                refs.append(ref)
                gots.append(out[b, h * self.G:(h + 1) * self.G])
        return check_outputs(np.array(gots), np.array(refs))

    def decode(self, qb):
        import torch
        dev = self.layer.device
        sel = torch.full((self.B, self.Hkv, self.kmax()), -7, dtype=torch.int32, device=dev)
        out = self.layer.decode(to_device_bf16(qb, dev), sel_out=sel)
        torch.cuda.synchronize()
        return out.cpu().numpy().astype(np.float64), sel.cpu().numpy()

    def decode_append(self, qb):
        import torch
        dev = self.layer.device
        kb, vb = self.new_tokens(1)
        sel = torch.full((self.B, self.Hkv, self.kmax()), -7, dtype=torch.int32, device=dev)
        out = self.layer.decode_append(to_device_bf16(qb, dev), to_device_bf16(np.ascontiguousarray(kb[:, :, 0]), dev),
                                       to_device_bf16(np.ascontiguousarray(vb[:, :, 0]), dev), sel_out=sel)
        torch.cuda.synchronize()
        res = out.cpu().numpy().astype(np.float64), sel.cpu().numpy()
        self.T = [t + 1 for t in self.T]
        return res

    def append_chunk(self, n):
        dev = self.layer.device
        kb, vb = self.new_tokens(n)
        self.layer.append_chunk(to_device_bf16(np.ascontiguousarray(kb), dev),
                                to_device_bf16(np.ascontiguousarray(vb), dev))
        self.T = [t + n for t in self.T]

    def random_q(self):
        return bf16_bits(self.rng.standard_normal((self.B, self.Hq, self.d)))

    def check_state(self):
        import torch
        L = self.layer
        L.sync_state()
        torch.cuda.synchronize()
        for b in range(self.B):
            for h in range(self.Hkv):
                T = self.T[b]
                K, V = self.K[b, h, :T], self.V[b, h, :T]
                part = O.partition(T, self.S, self.W[h], self.Bk)
                H, zk, zv, n = O.linear_state(K, V, part)
                mu, var = O.block_stats(K, part)
                assert float(L.n[b, h]) == n, (b, h)
                for name, ref, t in (("H", H, L.H[b, h]), ("zk", zk, L.zk[b, h]), ("zv", zv, L.zv[b, h]),
                                     ("mu", mu, L.mu[b, h, :part.nb]), ("var", var, L.var[b, h, :part.nb])):
                    if ref.size == 0:
                        continue
                    got = t.cpu().numpy().astype(np.float64)
                    den = np.linalg.norm(ref)
                    rel = np.linalg.norm(got - ref) / den if den > 0 else np.linalg.norm(got)
                    assert rel <= STATE_REL, (name, (b, h), rel)


def test_per_head_budgets_decode_steps_and_state():
    """Four KV heads with windows 64 / 128 / 300 / 1000 and top-k 2 / 8 / 0 / 5
    (one head exact over its window only); decode + append steps that cross
    block boundaries; the state of every unit after them."""
    c = RaggedCase(B=2, Hq=16, Hkv=4, d=128, row_T0=[3000, 3000], Bk=64, S=4,
                   head_W=[64, 128, 300, 1000], head_k=[2, 8, 0, 5], n_app=80, seed=3)
    q = c.random_q()
    out, sel = c.decode(q)
    c.check_decode(q, out, sel)
    for i in range(70):
        q = c.random_q()
        out, sel = c.decode_append(q)
        if i % 23 == 0:
            c.T = [t - 1 for t in c.T]      # the decode saw the length before its append
            c.check_decode(q, out, sel)
            c.T = [t + 1 for t in c.T]
    c.check_state()
    q = c.random_q()
    out, sel = c.decode(q)
    c.check_decode(q, out, sel)
    assert c.layer.status() == 0


def test_per_row_lengths_decode_steps_and_state():
    """Three rows at 4100, 1300 and 60 tokens (the last still inside sinks +
    window), uniform budget; decode + append steps; each row's output and state
    against the oracle at its own length."""
    c = RaggedCase(B=3, Hq=8, Hkv=2, d=64, row_T0=[4100, 1300, 60], Bk=32, S=4,
                   head_W=[64, 64], head_k=[4, 4], n_app=40, seed=5)
    q = c.random_q()
    out, sel = c.decode(q)
    c.check_decode(q, out, sel)
    for i in range(30):
        q = c.random_q()
        out, sel = c.decode_append(q)
        if i in (0, 9, 29):
            c.T = [t - 1 for t in c.T]
            c.check_decode(q, out, sel)
            c.T = [t + 1 for t in c.T]
    assert c.layer.row_lengths() == c.T
    c.check_state()
    assert c.layer.status() == 0


def test_rows_and_heads_with_chunked_appends_and_restore():
    """Per-row lengths and per-head budgets together; chunked appends (the
    dense fold of each unit's own pending evictions, none for a short row);
    the state, a decode, and a checkpoint restored with per-row lengths that
    decodes bit-identically."""
    import torch
    from hybrid_sparse_linear_decode_b200 import HybridAttentionLayer
    c = RaggedCase(B=2, Hq=8, Hkv=2, d=128, row_T0=[2500, 200], Bk=48, S=4,
                   head_W=[100, 256], head_k=[6, 3], n_app=220, seed=9)
    c.append_chunk(7)
    q = c.random_q()
    out, sel = c.decode(q)
    c.check_decode(q, out, sel)
    c.append_chunk(150)
    c.append_chunk(2)
    c.check_state()
    q = c.random_q()
    out, sel = c.decode(q)
    c.check_decode(q, out, sel)
    # checkpoint: synced state + caches + row lengths into fresh buffers
    c.layer.sync_state()
    torch.cuda.synchronize()
    L2 = HybridAttentionLayer(c.cfg, c.layer.device)
    for name in ("k_cache", "v_cache", "H", "zk", "zv", "n", "mu", "var"):
        getattr(L2, name).copy_(getattr(c.layer, name))
    L2.attach(c.layer.row_lengths())
    assert L2.row_lengths() == c.T
    dev = c.layer.device
    qd = to_device_bf16(c.random_q(), dev)
    s1 = torch.full((c.B, c.Hkv, c.kmax()), -7, dtype=torch.int32, device=dev)
    s2 = torch.full_like(s1, -7)
    o1 = c.layer.decode(qd, sel_out=s1)
    o2 = L2.decode(qd, sel_out=s2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)
    assert c.layer.status() == 0 and L2.status() == 0


def test_budget_and_row_arguments_are_checked():
    from hybrid_sparse_linear_decode_b200 import HybAttnError, HybridAttentionLayer, make_config
    import hybrid_sparse_linear_decode_b200 as H
    # a head's window below the config's window, a head's top-k above the config's top-k
    for hw, hk in (([32, 64], [2, 2]), ([64, 64], [2, 9])):
        cfg = make_config(1, 8, 2, 64, 32, 4, 64, 4, 1000, head_window=hw, head_top_k=hk)
        cfg.window, cfg.top_k = 64, 4
        with pytest.raises(HybAttnError):
            H.hyb_attn_query_sizes(cfg)
    cfg = make_config(2, 8, 2, 64, 32, 4, 64, 4, 1000)
    L = HybridAttentionLayer(cfg, "cuda")
    for rows in ([0, 100], [100, 1001]):
        with pytest.raises(HybAttnError):
            L.init(rows)
