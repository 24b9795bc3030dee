"""Host (numpy) side of the seeded input generator."""

import math

import numpy as np
import pytest

from syngen import configs as C
from syngen import host as H


def test_normal_matches_libm_box_muller():
    """The fixed-series ln / cos agree with libm's to ~1e-14: the generator is
    the Box-Muller transform, not some other distribution."""
    key = H.stream_key(3, 1)
    idx = np.arange(200_000, dtype=np.uint64)
    z = H.normal(key, idx)
    b = H.raw_bits(key, idx)
    hi = (b >> np.uint64(32)).astype(np.float64)
    lo = (b & np.uint64(0xFFFFFFFF)).astype(np.float64)
    ref = np.sqrt(-2 * np.log((hi + 1) * 2.0 ** -32)) * np.cos(2 * np.pi * lo * 2.0 ** -32)
    assert np.abs(z - ref).max() < 1e-13


def test_normal_moments():
    z = H.normal(H.stream_key(0, 2), np.arange(2_000_000, dtype=np.uint64))
    assert abs(z.mean()) < 3e-3
    assert abs(z.var() - 1) < 3e-3
    assert abs((z ** 3).mean()) < 1e-2
    assert abs((z ** 4).mean() - 3) < 2e-2


def test_streams_and_seeds_independent():
    idx = np.arange(100_000, dtype=np.uint64)
    a = H.normal(H.stream_key(0, 1), idx)
    b = H.normal(H.stream_key(0, 2), idx)
    c = H.normal(H.stream_key(1, 1), idx)
    assert abs(np.corrcoef(a, b)[0, 1]) < 0.01
    assert abs(np.corrcoef(a, c)[0, 1]) < 0.01
    assert not np.array_equal(a, c)


def test_bf16_rounding_matches_torch():
    """fp64 -> fp32 -> bf16 nearest-even, checked against torch's conversion."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100_000) * 10.0 ** rng.integers(-6, 6, 100_000),
                        np.array([0.0, -0.0, 1.0, -1.0, 65504.0, 1e-40])])
    got = H.f64_to_bf16_bits(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("name", ["tiny", "llama8b_32layers_b4_128k", "llama8b_32layers_b8_32k"])
def test_slices_are_consistent(name):
    """Any slice regenerates identically (counter-based): [t0, t1) of a long draw
    equals a fresh draw of [t0, t1)."""
    w = C.get_workload(name)
    tb = H.LayerTables(w, min(3, w.layers - 1))
    b, h = w.batch - 1, w.n_kv_heads - 1
    kb, vb = H.kv_bits(w, tb, b, h, 0, 300)
    k2, v2 = H.kv_bits(w, tb, b, h, 117, 260)
    assert np.array_equal(kb[117:260], k2) and np.array_equal(vb[117:260], v2)
    q0 = H.q_bits(w, 0, 0)
    assert q0.shape == (w.batch, w.n_q_heads, w.head_dim)
    assert np.array_equal(q0, H.q_bits(w, 0, 0))


def test_head_scale_recipe():
    w = C.get_workload("llama8b_32layers_b8_32k")
    s = H.head_scales(w)
    assert s.shape == (32, 8) and s.min() >= 0.5 and s.max() < 2.0
    assert abs(s.mean() - 1.25) < 0.15
    tb = H.LayerTables(w, 5)
    k, v = H.kv_f64(w, tb, 2, 3, 0, 4000)
    assert abs(k.std() / tb.scale[3] - 1) < 0.03 and abs(v.std() / tb.scale[3] - 1) < 0.03


def test_block_offset_recipe():
    """Per-block key offset N(0, 0.5^2), constant over a block, none on sinks."""
    w = C.get_workload("llama8b_32layers_b4_128k")
    tb = H.LayerTables(w, 0)
    k, _ = H.kv_f64(w, tb, 1, 2, 0, w.n_sink + 64 * 200)
    blocks = k[w.n_sink:].reshape(200, 64, -1)
    means = blocks.mean(axis=1)                       # ~ offset + N(0, 1/64)
    assert abs(means.std() - math.sqrt(0.25 + 1 / 64)) < 0.03
    assert abs(k[:w.n_sink].std() - 1) < 0.25


def test_planted_recipe():
    """Planted blocks hold keys 3 * q_hat + N(0, 0.1^2), q_hat the unit vector
    of the group-summed step-0 query."""
    w = C.get_workload("tiny")
    tb = H.LayerTables(w, 0)
    P = tb.planted[0, 0]
    assert len(P) == 2 and len(set(P.tolist())) == 2
    k, _ = H.kv_f64(w, tb, 0, 0, 0, w.T0)
    for j in P:
        a = w.n_sink + j * w.block_size
        blk = k[a:a + w.block_size]
        np.testing.assert_allclose(blk.mean(axis=0), 3 * tb.qhat[0, 0], atol=0.06)
        assert abs(blk.std(axis=0).mean() - 0.1) < 0.02
    assert abs(np.linalg.norm(tb.qhat[0, 0]) - 1) < 1e-12


def test_tiny_oracle_selects_planted_blocks():
    """On the tiny workload the second-order score separates the planted blocks
    (group score ~ 6) from the background (~ 2 +- 0.4), so the oracle's top-4
    contains both planted blocks."""
    import oracle as O
    w = C.get_workload("tiny")
    tb = H.LayerTables(w, 0)
    K, V = H.kv_f64(w, tb, 0, 0, 0, w.T0)
    q = H.bf16_bits_to_f64(H.q_bits(w, 0, 0))[0]
    u = O.OracleUnit(K, V, w.n_sink, w.window, w.block_size, w.top_k, 1 / math.sqrt(w.head_dim))
    out, sel, scores = u.decode(q)
    assert set(tb.planted[0, 0].tolist()) <= set(sel.tolist())
    assert scores[tb.planted[0, 0]].min() > 4.5
    bg = np.delete(scores, tb.planted[0, 0])
    assert 1.0 < bg.mean() < 3.0


def test_layer_budgets_view():
    """A workload with per-layer budgets gives each layer its own (top_k,
    window), cycled over the layers; one without gives every layer itself."""
    from syngen import configs as C
    w = C.get_workload("llama8b_32layers_b8_32k_budgets")
    for l in range(w.layers):
        v = w.for_layer(l)
        assert (v.top_k, v.window) == w.layer_budgets[l % len(w.layer_budgets)]
        assert v.layer_budgets == () and v.T0 == w.T0 and v.capacity == w.capacity
    base = C.get_workload("llama8b_32layers_b8_32k")
    assert base.for_layer(5) is base


def test_algorithmic_bytes_match_the_per_head_figures():
    """The benchmark's algorithmic bytes per (layer, b) at the workloads' prefill
    length, against the method's per-KV-head bytes written out by hand: exact
    KV 2052 x 128 x 4, statistics nb x 2 x 128 x 4, state (128^2 + 2 x 128 + 1) x 4,
    q + out 4 x 128 x 6."""
    import bench
    from syngen import configs as C
    w = C.get_workload("llama8b_32k_layer")
    dec, _ = bench.algorithmic_bytes(w, w.T0)
    assert w.n_blocks(w.T0) == 496 and w.exact_tokens(w.T0) == 2052
    assert dec == 1_050_624 + 507_904 + 66_564 + 3_072
    assert dec * w.n_kv_heads == 13_025_312
    w4 = C.get_workload("llama8b_32layers_b4_128k")
    dec4, _ = bench.algorithmic_bytes(w4, w4.T0)
    assert dec4 * w4.n_kv_heads == 33_865_760
