"""Shared helpers of the GPU parity tests: build a layer from host-generated
bf16 inputs, run the CUDA path through the C ABI, and compare with the fp64
oracle (which sees only the same host-generated inputs).

Tolerances (the parity bar):
* selection: identical, except that a block may differ when its oracle score
  is within 1e-4 * max(1, |score_k|) of the oracle's k-th largest score;
* outputs (oracle given the GPU's selection): max |a - b| <= 2e-3 and
  ||a - b||_2 / ||b||_2 <= 5e-3 over the whole output tensor;
* state (H, zk, zv, n, mu, var): ||a - b||_2 / ||b||_2 <= 1e-4 per tensor and
  per unit.
"""

from __future__ import annotations

import math

import numpy as np

import oracle as O
from syngen import host as SH

OUT_MAX_ABS = 2e-3
OUT_REL_L2 = 5e-3
SEL_TIE = 1e-4
STATE_REL = 1e-4


def bf16_bits(x: np.ndarray) -> np.ndarray:
    return SH.f64_to_bf16_bits(x)


def bits_to_f64(b: np.ndarray) -> np.ndarray:
    return SH.bf16_bits_to_f64(b)


def to_device_bf16(bits: np.ndarray, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


class Case:
    """A layer with random (or given) bf16 history on the host and the device."""

    def __init__(self, B, Hq, Hkv, d, T0, Bk, S, W, k, n_append=0, seed=0, device="cuda", scale=0.0,
                 kv_bits=None, k_scale=1.0, capacity=None):
        import torch
        from hybrid_sparse_linear_decode_b200 import HybridAttentionLayer, make_config
        self.B, self.Hq, self.Hkv, self.d = B, Hq, Hkv, d
        self.G = Hq // Hkv
        self.S, self.W, self.Bk, self.k = S, W, Bk, k
        self.T0 = T0
        self.scale = scale if scale > 0 else 1.0 / math.sqrt(d)
        total = T0 + n_append
        rng = np.random.default_rng(seed)
        if kv_bits is None:
            Kb = bf16_bits(rng.standard_normal((B, Hkv, total, d)) * k_scale)
            Vb = bf16_bits(rng.standard_normal((B, Hkv, total, d)))
        else:
            Kb, Vb = kv_bits
        self.Kb, self.Vb = Kb, Vb
        self.K, self.V = bits_to_f64(Kb), bits_to_f64(Vb)
        self.rng = rng
        cap = capacity or max(total, 1)
        self.cfg = make_config(B, Hq, Hkv, d, Bk, S, W, k, cap, scale)
        self.layer = HybridAttentionLayer(self.cfg, device)
        dev = self.layer.device
        if T0 > 0:
            self.layer.k_cache[:, :, :T0].copy_(to_device_bf16(Kb[:, :, :T0], dev))
            self.layer.v_cache[:, :, :T0].copy_(to_device_bf16(Vb[:, :, :T0], dev))
        self.layer.init(T0)
        self.T = T0
        torch.cuda.synchronize()

    def random_q(self):
        return bf16_bits(self.rng.standard_normal((self.B, self.Hq, self.d)))

    def append(self, n=1):
        for _ in range(n):
            t = self.T
            kb = to_device_bf16(np.ascontiguousarray(self.Kb[:, :, t]), self.layer.device)
            vb = to_device_bf16(np.ascontiguousarray(self.Vb[:, :, t]), self.layer.device)
            self.layer.append(kb, vb)
            self.T += 1
        assert self.layer.T == self.T

    def decode(self, q_bits, with_scores=True):
        import torch
        dev = self.layer.device
        q = to_device_bf16(q_bits, dev)
        sel = torch.full((self.B, self.Hkv, self.k), -7, dtype=torch.int32, device=dev)
        mb = max(1, self.layer.sizes.max_blocks)
        scores = torch.zeros((self.B, self.Hkv, mb), dtype=torch.float32, device=dev) if with_scores else None
        out = self.layer.decode(q, sel_out=sel, scores_out=scores)
        torch.cuda.synchronize()
        return (out.cpu().numpy().astype(np.float64), sel.cpu().numpy(),
                None if scores is None else scores.cpu().numpy())

    def decode_with_selection(self, q_bits, sel_np):
        import torch
        dev = self.layer.device
        q = to_device_bf16(q_bits, dev)
        sel = torch.from_numpy(np.ascontiguousarray(sel_np, dtype=np.int32)).to(dev)
        out = self.layer.decode_with_selection(q, sel)
        torch.cuda.synchronize()
        return out.cpu().numpy().astype(np.float64)

    # ---- oracle side -------------------------------------------------------
    def unit_kv(self, b, h, T=None):
        T = self.T if T is None else T
        return self.K[b, h, :T], self.V[b, h, :T]

    def oracle_unit(self, q_bits, b, h, sel=None):
        """(out [G, d], sel, scores) of the oracle for unit (b, h) at the current T."""
        K, V = self.unit_kv(b, h)
        part = O.partition(self.T, self.S, self.W, self.Bk)
        q = bits_to_f64(q_bits)[b, h * self.G:(h + 1) * self.G]
        mu, var = O.block_stats(K, part)
        scores = O.block_scores(q, mu, var, self.scale) if part.nb else np.zeros(0)
        osel = O.select_blocks(scores, self.k)
        use = osel if sel is None else sel
        out = O.hybrid_subtract(q, K, V, part, use, self.scale)
        return out, osel, scores

    def state_gpu(self):
        import torch
        L = self.layer
        L.sync_state()  # fold the evictions since the last decode
        torch.cuda.synchronize()
        return {n: getattr(L, n).cpu().numpy().astype(np.float64) for n in ("H", "zk", "zv", "n", "mu", "var")}


def check_selection(gpu_sel_row, oracle_scores, k):
    """GPU selection row (int32 [k], -1 padded) against the oracle scores."""
    nb = oracle_scores.shape[0]
    ke = min(k, nb)
    g = [int(j) for j in gpu_sel_row]
    assert all(j == -1 for j in g[ke:]), g
    got = g[:ke]
    assert got == sorted(got) and len(set(got)) == ke and all(0 <= j < nb for j in got), got
    if ke == 0:
        return 0
    osel = O.select_blocks(oracle_scores, k)
    kth = np.sort(oracle_scores)[::-1][ke - 1]
    diff = set(got) ^ set(int(j) for j in osel)
    tol = SEL_TIE * max(1.0, abs(kth))
    for j in diff:
        assert abs(oracle_scores[j] - kth) <= tol, (j, oracle_scores[j], kth, sorted(got), list(osel))
    return len(diff)


def check_outputs(gpu, ref, max_abs=OUT_MAX_ABS, rel_l2=OUT_REL_L2):
    err = np.abs(gpu - ref)
    rel = np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-30)
    assert np.all(np.isfinite(gpu))
    assert err.max() <= max_abs, f"max abs err {err.max():.3e}"
    assert rel <= rel_l2, f"rel L2 err {rel:.3e}"
    return err.max(), rel


def check_state(case: Case, units=None):
    """GPU state after init/appends against the oracle's direct definition."""
    st = case.state_gpu()
    part = O.partition(case.T, case.S, case.W, case.Bk)
    worst = 0.0
    units = units or [(b, h) for b in range(case.B) for h in range(case.Hkv)]
    for (b, h) in units:
        K, V = case.unit_kv(b, h)
        H, zk, zv, n = O.linear_state(K, V, part)
        mu, var = O.block_stats(K, part)
        assert st["n"][b, h] == n
        for name, ref, got in (("H", H, st["H"][b, h]), ("zk", zk, st["zk"][b, h]), ("zv", zv, st["zv"][b, h]),
                               ("mu", mu, st["mu"][b, h, :part.nb]), ("var", var, st["var"][b, h, :part.nb])):
            if ref.size == 0:
                continue
            den = np.linalg.norm(ref)
            rel = np.linalg.norm(got - ref) / den if den > 0 else np.linalg.norm(got)
            assert rel <= STATE_REL, f"{name} unit {(b, h)} rel {rel:.3e}"
            worst = max(worst, rel)
    return worst


def full_check(case: Case, q_bits, units=None, check_scores=True):
    """Decode once; check selection, scores, outputs for the given units (all by default)."""
    out, sel, scores = case.decode(q_bits)
    units = units or [(b, h) for b in range(case.B) for h in range(case.Hkv)]
    refs, gots = [], []
    for (b, h) in units:
        ref_out, osel, oscores = case.oracle_unit(q_bits, b, h, sel=None)
        check_selection(sel[b, h], oscores, case.k)
        if check_scores and oscores.size:
            np.testing.assert_allclose(scores[b, h, :oscores.size], oscores, rtol=1e-4, atol=1e-4)
        gsel = [int(j) for j in sel[b, h] if j >= 0]
        ref_gsel, _, _ = case.oracle_unit(q_bits, b, h, sel=np.array(gsel, dtype=np.int64))
        refs.append(ref_gsel)
        gots.append(out[b, h * case.G:(h + 1) * case.G])
    return check_outputs(np.array(gots), np.array(refs)), sel
