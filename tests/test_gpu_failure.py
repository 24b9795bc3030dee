"""Failure detection and checkpoint / restore on the GPU, in forms that fault,
trap or hang nothing: a bounded wait made to run out by withholding a hand-off
(a flag that nothing else sets), host-written non-finite inputs, inputs that
drive the shared normaliser below zero, and a checkpoint copied into fresh
buffers and attached without rebuilding the state."""

import numpy as np
import pytest

from harness import Case, bf16_bits, check_outputs, full_check, to_device_bf16
import oracle as O

pytestmark = pytest.mark.gpu


def _case(**kw):
    base = dict(B=1, Hq=4, Hkv=1, d=128, T0=4 + 64 + 32 * 100, Bk=32, S=4, W=64, k=4, n_append=0, seed=21)
    base.update(kw)
    return Case(**base)


def test_withheld_scores_make_the_bounded_wait_run_out_and_the_context_recovers():
    """One unit, so a cluster of up to 16 ranks scores 100 blocks; rank 1
    withholds its share.  Every other rank's wait for the scores gives up after
    the 20 ms limit and the status word says so; the launch returns.  With the
    flag cleared the same context decodes correctly again."""
    import torch
    from hybrid_sparse_linear_decode_b200 import HYB_STATUS_TIMEOUT, HYB_TEST_WITHHOLD_SCORES
    c = _case()
    L = c.layer
    assert L.status(clear=True) == 0
    L.set_wait_limit(20_000_000)
    L.set_test_flags(HYB_TEST_WITHHOLD_SCORES)
    c.decode(c.random_q())
    torch.cuda.synchronize()
    assert L.status(clear=True) & HYB_STATUS_TIMEOUT
    L.set_test_flags(0)
    L.set_wait_limit(0)
    full_check(c, c.random_q())
    assert L.status() == 0


def test_wait_limit_bounds_are_checked():
    from hybrid_sparse_linear_decode_b200 import HybAttnError
    c = _case(T0=600)
    for bad in (1, 99_999, 60_000_000_001):
        with pytest.raises(HybAttnError):
            c.layer.set_wait_limit(bad)
    with pytest.raises(HybAttnError):
        c.layer.set_test_flags(0x80)
    c.layer.set_wait_limit(100_000)
    c.layer.set_wait_limit(0)


def test_nan_in_q_is_reported():
    """A NaN written by the host into one query head: its group's scores are NaN
    (ranked last) and its outputs are not finite; both are reported."""
    from hybrid_sparse_linear_decode_b200 import HYB_STATUS_NAN_SCORE, HYB_STATUS_NONFINITE
    c = _case(T0=1500)
    q = c.random_q()
    q[0, 2, 5] = 0x7FC0    # bf16 quiet NaN
    c.decode(q)
    st = c.layer.status(clear=True)
    assert st & HYB_STATUS_NONFINITE and st & HYB_STATUS_NAN_SCORE
    full_check(c, c.random_q())
    assert c.layer.status() == 0


def test_nonpositive_normaliser_is_reported():
    """No sinks, no window, no selected block: every token takes the Taylor
    weight 1 + s.  Keys opposite to the query make s far below -1, so the
    shared normaliser is negative; it is not clamped (the output is what the
    definition gives) and the status word reports it."""
    from hybrid_sparse_linear_decode_b200 import HYB_STATUS_DENOMINATOR
    B, Hkv, d, T0 = 1, 1, 64, 200
    rng = np.random.default_rng(4)
    Kf = -2.0 + 0.01 * rng.standard_normal((B, Hkv, T0, d))
    Vf = rng.standard_normal((B, Hkv, T0, d))
    c = Case(B, 4, Hkv, d, T0, 16, 0, 0, 0, kv_bits=(bf16_bits(Kf), bf16_bits(Vf)))
    q = bf16_bits(np.full((1, 4, d), 2.0))
    out, _, _ = c.decode(q)
    assert c.layer.status(clear=True) & HYB_STATUS_DENOMINATOR
    ref = O.pure_taylor(np.full((4, d), 2.0), c.K[0, 0], c.V[0, 0], T0, c.scale)
    assert (1.0 + (np.full((4, d), 2.0) * c.scale) @ c.K[0, 0].T).sum(axis=1).max() < 0
    check_outputs(out[0], ref, max_abs=2e-3 * np.abs(ref).max(), rel_l2=5e-3)


def _clone_layer(src):
    """Fresh buffers holding a copy of every state and cache array of `src`."""
    from hybrid_sparse_linear_decode_b200 import HybridAttentionLayer
    dst = HybridAttentionLayer(src.cfg, src.device)
    for name in ("k_cache", "v_cache", "H", "zk", "zv", "n", "mu", "var"):
        getattr(dst, name).copy_(getattr(src, name))
    return dst


def test_checkpoint_restore_gives_an_identical_decode():
    """Checkpoint = state synced, then caches + state arrays + T copied.  A
    context attached to the copy decodes bit-identically to the original, and
    both stay identical through further decode + append steps."""
    import torch
    c = _case(B=2, Hq=16, Hkv=4, T0=1500, Bk=64, W=100, k=6, n_append=12, seed=8)
    for _ in range(5):           # some history: decodes folding appends
        c.decode(c.random_q())
        c.append()
    c.layer.sync_state()
    torch.cuda.synchronize()
    L2 = _clone_layer(c.layer)
    L2.attach(c.T)
    assert L2.T == c.layer.T == c.T
    dev = c.layer.device
    for i in range(4):
        q = to_device_bf16(c.random_q(), dev)
        kb = to_device_bf16(np.ascontiguousarray(c.Kb[:, :, c.T]), dev)
        vb = to_device_bf16(np.ascontiguousarray(c.Vb[:, :, c.T]), dev)
        s1 = torch.full((c.B, c.Hkv, c.k), -7, dtype=torch.int32, device=dev)
        s2 = torch.full_like(s1, -7)
        o1 = c.layer.decode_append(q, kb, vb, sel_out=s1)
        o2 = L2.decode_append(q, kb, vb, sel_out=s2)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(s1, s2), i
        c.T += 1
    assert c.layer.status() == 0 and L2.status() == 0
    full_check(c, c.random_q())
