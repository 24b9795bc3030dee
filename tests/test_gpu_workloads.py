"""Parity at the full sizes of the synthetic workloads, in the launch
configuration the benchmark times: device caches are filled by the device
generator, the oracle regenerates the same units on the host (bit-identical
generator twins, see test_gpu_syngen.py) for sampled units."""

import math

import numpy as np
import pytest

import oracle as O
from harness import bits_to_f64, check_outputs, check_selection, to_device_bf16, OUT_MAX_ABS, OUT_REL_L2, SEL_TIE, STATE_REL
from syngen import configs as C
from syngen import host as SH

pytestmark = pytest.mark.gpu


class WorkloadLayer:
    def __init__(self, w: C.Workload, layer: int, device="cuda", n_app=None):
        import torch
        import syngen.device as SD
        from hybrid_sparse_linear_decode_b200 import HybridAttentionLayer, make_config
        SD.build()
        w = w.for_layer(layer)  # the layer's own top-k and window when budgets vary by layer
        self.w, self.l = w, layer
        self.n_app = w.capacity - w.T0 if n_app is None else n_app
        heads = [w.for_head(h) for h in range(w.n_kv_heads)]  # per-head budgets, when the workload has them
        self.k_max = max(wh.top_k for wh in heads)
        cfg = make_config(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.block_size, w.n_sink,
                          min(wh.window for wh in heads), self.k_max, w.T0 + self.n_app,
                          head_window=[wh.window for wh in heads] if w.head_budgets else None,
                          head_top_k=[wh.top_k for wh in heads] if w.head_budgets else None)
        self.layer = HybridAttentionLayer(cfg, device)
        self.tables = SD.DeviceTables(w, layer, self.layer.device)
        SD.fill_kv(w, self.tables, self.layer.k_cache, self.layer.v_cache, 0, w.T0)
        self.app_k = self.app_v = None
        if self.n_app:
            shp = (w.batch, w.n_kv_heads, self.n_app, w.head_dim)
            self.app_k = torch.empty(shp, dtype=torch.bfloat16, device=self.layer.device)
            self.app_v = torch.empty(shp, dtype=torch.bfloat16, device=self.layer.device)
            SD.fill_kv(w, self.tables, self.app_k, self.app_v, w.T0, w.T0 + self.n_app, t_out0=w.T0)
        self.layer.init(w.T0)
        self.T = w.T0
        self.scale = 1 / math.sqrt(w.head_dim)
        self._host = {}

    def q_bits(self, step):
        return SH.q_bits(self.w, self.l, step)

    def decode(self, qb):
        import torch
        dev = self.layer.device
        sel = torch.full((self.w.batch, self.w.n_kv_heads, self.k_max), -7, dtype=torch.int32, device=dev)
        out = self.layer.decode(to_device_bf16(qb, dev), sel_out=sel)
        torch.cuda.synchronize()
        return out.cpu().numpy().astype(np.float64), sel.cpu().numpy()

    def append(self, i):
        self.layer.append(self.app_k[:, :, i].contiguous(), self.app_v[:, :, i].contiguous())
        self.T += 1

    def host_unit(self, b, h):
        if (b, h) not in self._host:
            self._host[(b, h)] = SH.kv_f64(self.w, self.tables.host, b, h, 0, self.w.T0 + self.n_app)
        return self._host[(b, h)]

    def check_units(self, qb, units, out, sel):
        w = self.w
        G = w.group
        refs, gots, ndiff = [], [], 0
        for (b, h) in units:
            wh = w.for_head(h)  # the head's own budget
            part = O.partition(self.T, w.n_sink, wh.window, w.block_size)
            K, V = self.host_unit(b, h)
            K, V = K[:self.T], V[:self.T]
            q = bits_to_f64(qb)[b, h * G:(h + 1) * G]
            mu, var = O.block_stats(K, part)
            scores = O.block_scores(q, mu, var, self.scale)
            assert all(j == -1 for j in sel[b, h][wh.top_k:])
            ndiff += check_selection(sel[b, h][:wh.top_k], scores, wh.top_k)
            gsel = np.array([j for j in sel[b, h] if j >= 0])
            refs.append(O.hybrid_subtract(q, K, V, part, gsel, self.scale))
            gots.append(out[b, h * G:(h + 1) * G])
        return check_outputs(np.array(gots), np.array(refs)), ndiff

    def check_state(self, units):
        w = self.w
        L = self.layer
        L.sync_state()  # fold the evictions since the last decode
        for (b, h) in units:
            part = O.partition(self.T, w.n_sink, w.for_head(h).window, w.block_size)
            K, V = self.host_unit(b, h)
            K, V = K[:self.T], V[:self.T]
            H, zk, zv, n = O.linear_state(K, V, part)
            mu, var = O.block_stats(K, part)
            assert float(L.n[b, h]) == n
            for name, ref, t in (("H", H, L.H[b, h]), ("zk", zk, L.zk[b, h]), ("zv", zv, L.zv[b, h]),
                                 ("mu", mu, L.mu[b, h, :part.nb]), ("var", var, L.var[b, h, :part.nb])):
                got = t.cpu().numpy().astype(np.float64)
                rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
                assert rel <= STATE_REL, (name, (b, h), rel)


def test_tiny_workload_decode_appends_state():
    w = C.get_workload("tiny")
    wl = WorkloadLayer(w, 0)
    units = [(0, 0)]
    qb = wl.q_bits(0)
    out, sel = wl.decode(qb)
    (mx, rel), nd = wl.check_units(qb, units, out, sel)
    planted = set(wl.tables.host.planted[0, 0].tolist())
    assert planted <= set(sel[0, 0].tolist())
    for i in range(w.appends_after_decode):
        wl.append(i)
    wl.check_state(units)
    qb = SH.q_bits(w, 0, 1)
    out, sel = wl.decode(qb)
    wl.check_units(qb, units, out, sel)


def test_llama8b_32k_layer_every_unit():
    w = C.get_workload("llama8b_32k_layer")
    wl = WorkloadLayer(w, 0, n_app=0)
    units = [(0, h) for h in range(w.n_kv_heads)]
    qb = wl.q_bits(0)
    out, sel = wl.decode(qb)
    wl.check_units(qb, units, out, sel)
    wl.check_state(units)
    # every planted block is selected
    for h in range(w.n_kv_heads):
        assert set(wl.tables.host.planted[0, h].tolist()) <= set(sel[0, h].tolist())
    # q = 0 at full size: the mean of V over [0, T) for every unit
    out0, _ = wl.decode(np.zeros_like(qb))
    for h in range(2):
        _, V = wl.host_unit(0, h)
        check_outputs(out0[0, h * w.group:(h + 1) * w.group],
                      np.broadcast_to(V[:w.T0].mean(axis=0), (w.group, w.head_dim)), max_abs=1e-4, rel_l2=1e-4)


@pytest.mark.parametrize("layer", [0, 31])
def test_llama8b_32layers_b8_32k_sampled(layer):
    w = C.get_workload("llama8b_32layers_b8_32k")
    wl = WorkloadLayer(w, layer, n_app=1)
    # the layer's KV heads with the smallest and the largest scale (U(0.5, 2)),
    # at both batch ends, and two more
    sc = SH.head_scales(w)[layer]
    lo, hi = int(np.argmin(sc)), int(np.argmax(sc))
    rest = [h for h in range(w.n_kv_heads) if h not in (lo, hi)]
    units = [(0, lo), (7, hi), (3, rest[0]), (5, rest[-1])]
    qb = wl.q_bits(0)
    out, sel = wl.decode(qb)
    wl.check_units(qb, units, out, sel)
    wl.append(0)
    wl.check_state(units[:2])


@pytest.mark.parametrize("layer", [0, 1, 2, 3])
def test_llama8b_32layers_b8_32k_budgets_sampled(layer):
    """Per-layer budgets: each layer its own top-k and window (k 8..32, W
    512..2048), decoded, appended and checked against the oracle with that
    layer's budget."""
    w = C.get_workload("llama8b_32layers_b8_32k_budgets")
    wl = WorkloadLayer(w, layer, n_app=1)
    assert (wl.w.top_k, wl.w.window) == w.layer_budgets[layer]
    units = [(0, 0), (4, 6), (7, 3)]
    qb = wl.q_bits(0)
    out, sel = wl.decode(qb)
    assert sel.shape[-1] == wl.w.top_k
    wl.check_units(qb, units, out, sel)
    wl.append(0)
    wl.check_state(units[:2])


@pytest.mark.parametrize("layer,units", [
    (9, [(0, 0), (0, 7), (3, 0), (3, 7), (1, 4)]),     # both batch ends, both ends of the KV heads
    (22, [(0, 3), (3, 2), (2, 6), (1, 1), (2, 0)]),
])
def test_llama8b_32layers_b4_128k_sampled(layer, units):
    """Ten units over two layers of the 128K workload: every unit's keys carry
    its own per-block offsets, so the sample spans the offset regime; selection
    above 512 blocks (2016 candidates, k = 32)."""
    w = C.get_workload("llama8b_32layers_b4_128k")
    wl = WorkloadLayer(w, layer, n_app=0)
    qb = wl.q_bits(0)
    out, sel = wl.decode(qb)
    wl.check_units(qb, units, out, sel)
    assert wl.layer.status() == 0


def test_llama8b_32layers_b8_32k_head_budgets_sampled():
    """Per-KV-head budgets at full size: the 8 KV heads of a layer cycle through
    (k, W) = (8, 512), (16, 1024), (24, 1536), (32, 2048); units of every budget
    and both batch ends against the oracle with their own head's budget, then
    the state after an append."""
    w = C.get_workload("llama8b_32layers_b8_32k_head_budgets")
    wl = WorkloadLayer(w, 5, n_app=1)
    units = [(0, 0), (7, 1), (3, 2), (5, 3), (1, 7)]
    qb = wl.q_bits(0)
    out, sel = wl.decode(qb)
    wl.check_units(qb, units, out, sel)
    wl.append(0)
    wl.check_state(units[:2])
    assert wl.layer.status() == 0


def test_llama8b_32k_layer_tokens_every_unit():
    """Token-granular exact set at full size: blocks of one token (31.7 K
    candidates per unit), the top 1024 tokens exact; every unit against the
    oracle."""
    w = C.get_workload("llama8b_32k_layer_tokens")
    wl = WorkloadLayer(w, 0, n_app=0)
    qb = wl.q_bits(0)
    out, sel = wl.decode(qb)
    wl.check_units(qb, [(0, h) for h in range(w.n_kv_heads)], out, sel)
    assert wl.layer.status() == 0


def test_llama8b_32layers_b8_32k_strided_sampled():
    """Strided block selection at full size (stride 16 over 496 candidate
    blocks: 31 always-exact blocks, plus the top 16 of the others), in the
    bench's configuration: the selection row sized for the union."""
    import torch
    from hybrid_sparse_linear_decode_b200 import HybridAttentionLayer, make_config
    import syngen.device as SD
    w = C.get_workload("llama8b_32layers_b8_32k")
    stride, k_top = 16, 16
    nb = w.n_blocks(w.T0)
    width = nb // stride + min(k_top, nb - nb // stride)
    SD.build()
    cfg = make_config(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.block_size, w.n_sink, w.window, width, w.T0)
    L = HybridAttentionLayer(cfg, "cuda")
    tables = SD.DeviceTables(w, 3, L.device)
    SD.fill_kv(w, tables, L.k_cache, L.v_cache, 0, w.T0)
    L.init(w.T0)
    qb = SH.q_bits(w, 3, 0)
    sel = torch.full((w.batch, w.n_kv_heads, width), -7, dtype=torch.int32, device=L.device)
    out = L.decode_strided(to_device_bf16(qb, L.device), k_top, stride, sel_out=sel)
    torch.cuda.synchronize()
    out, sel = out.cpu().numpy().astype(np.float64), sel.cpu().numpy()
    assert L.status() == 0
    scale = 1 / math.sqrt(w.head_dim)
    part = O.partition(w.T0, w.n_sink, w.window, w.block_size)
    refs, gots = [], []
    for (b, h) in [(0, 0), (7, 7), (3, 5)]:
        K, V = SH.kv_f64(w, tables.host, b, h, 0, w.T0)
        q = bits_to_f64(qb)[b, h * w.group:(h + 1) * w.group]
        mu, var = O.block_stats(K, part)
        scores = O.block_scores(q, mu, var, scale)
        want = set(int(j) for j in O.select_blocks_strided(scores, k_top, stride))
        got = [int(j) for j in sel[b, h]]
        assert got == sorted(got) and len(got) == width and set(O.strided_blocks(part.nb, stride)) <= set(got)
        fixed = set(int(j) for j in O.strided_blocks(part.nb, stride))
        others = np.sort(np.array([scores[j] for j in range(part.nb) if j not in fixed]))[::-1]
        kth = others[k_top - 1]
        for j in set(got) ^ want:
            assert abs(scores[j] - kth) <= SEL_TIE * max(1.0, abs(kth)), (j, scores[j], kth)
        refs.append(O.hybrid_subtract(q, K, V, part, np.array(got, dtype=np.int64), scale))
        gots.append(out[b, h * w.group:(h + 1) * w.group])
    check_outputs(np.array(gots), np.array(refs))


def test_llama8b_256k_256_steps_every_unit():
    """All 8 units of the 256K workload at steps 0, 97 and 255 of 256 decode +
    append steps, and the state of every unit after the 256 appends."""
    w = C.get_workload("llama8b_256k_256steps")
    wl = WorkloadLayer(w, 0)
    assert wl.n_app == 256
    units = [(0, h) for h in range(w.n_kv_heads)]
    for step in range(w.steps):
        qb = wl.q_bits(step)
        out, sel = wl.decode(qb)
        if step in (0, 97, 255):
            wl.check_units(qb, units, out, sel)
            for h in range(w.n_kv_heads):
                if step == 0:
                    assert set(wl.tables.host.planted[0, h].tolist()) <= set(sel[0, h].tolist())
        wl.append(step)
    assert wl.layer.T == w.T0 + 256
    wl.check_state(units)
    assert wl.layer.status() == 0
