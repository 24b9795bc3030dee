"""GPU parity of the CUDA path (through the C ABI) against the fp64 oracle, at
sizes the oracle finishes in seconds: several tiles, ragged tails and the
degenerate cases of the method."""

import math

import numpy as np
import pytest

from harness import Case, check_outputs, check_selection, check_state, full_check, bits_to_f64
import oracle as O

pytestmark = pytest.mark.gpu


def _case(**kw):
    base = dict(B=1, Hq=4, Hkv=1, d=128, T0=600, Bk=32, S=4, W=64, k=4, n_append=0, seed=1)
    base.update(kw)
    return Case(**base)


@pytest.mark.parametrize("kw", [
    dict(),                                                   # plain
    dict(d=64),                                               # head dim 64
    dict(Hq=2, Hkv=1), dict(Hq=8, Hkv=8),                     # G = 2, G = 1
    dict(B=2, Hq=16, Hkv=4, T0=1500),                         # several units
    dict(T0=3, S=4, W=16),                                    # T <= S: sinks only
    dict(T0=15, S=4, W=16),                                   # S < T <= S + W: no evicted token
    dict(T0=4 + 16 + 30, S=4, W=16, Bk=8, k=8),               # nb <= k: every block selected
    dict(T0=4 + 64 + 32 * 5 + 1),                             # newest block holds 1 token
    dict(k=0),                                                # nothing selected
    dict(W=0),                                                # no window
    dict(S=0),                                                # no sinks
    dict(S=0, W=0, k=0, T0=333),                              # empty exact set: pure Taylor
    dict(Bk=100, k=3, T0=1200),                               # block spans 2 chunks, ragged
    dict(Bk=128, k=5, T0=2000, W=200),                        # 2 chunks per block
    dict(Bk=200, k=2, T0=1500, W=70),                         # 4 chunks per block, partial pieces
    dict(Bk=16, k=30, T0=1000, W=100),                        # many short blocks
    dict(W=1000, T0=3000, S=7),                               # long unaligned window
    dict(B=4, Hq=32, Hkv=8, T0=5000, Bk=64, W=1024, k=16),    # 32 units, CTAs span units
    dict(scale=0.05),                                         # explicit scale
    dict(k_scale=3.0, T0=900),                                # large scores (max shift matters)
])
def test_decode_matches_oracle(kw):
    c = _case(**kw)
    q = c.random_q()
    (mx, rel), _ = full_check(c, q)
    assert c.layer.status() == 0


def test_all_selected_is_softmax_and_q0_is_mean():
    """Closed-form properties through the GPU: k >= nb gives full softmax;
    q = 0 gives the mean of V over [0, T)."""
    c = _case(T0=700, Bk=32, k=1000, W=64)
    q = c.random_q()
    out, sel, _ = c.decode(q)
    Kf, Vf = c.unit_kv(0, 0)
    ref = O.full_softmax(bits_to_f64(q)[0], Kf, Vf, c.T, c.scale)
    check_outputs(out[0], ref)
    out0, _, _ = c.decode(np.zeros_like(q))
    check_outputs(out0[0], np.broadcast_to(Vf.mean(axis=0), out0[0].shape), max_abs=1e-4, rel_l2=1e-4)


@pytest.mark.parametrize("kw,n", [
    (dict(T0=600, Bk=32, W=64), 40),
    (dict(T0=4 + 64 + 32 * 3, Bk=32, W=64), 3),               # the first append opens a new block
    (dict(T0=601, Bk=32, W=64), 2),                           # two pending: folded inside the decode kernel
    (dict(T0=601, Bk=32, W=64), 4),                           # four pending: folded inside the decode kernel
    (dict(T0=601, Bk=32, W=64), 5),                           # five pending: the dense fold pass
    (dict(T0=10, S=4, W=16, Bk=8), 40),                       # grows from sinks-only through eviction
    (dict(T0=200, W=0, Bk=8), 20),                            # W = 0 evicts the appended token itself
    (dict(T0=300, S=0, W=5, Bk=7, d=64), 30),
    (dict(B=2, Hq=8, Hkv=2, T0=900, Bk=100, W=50), 110),      # fills a whole 100-token block
])
def test_append_state_and_decode(kw, n):
    """State after n appends equals the direct definition on the final history,
    and decode after the appends still matches the oracle."""
    c = _case(n_append=n, **kw)
    check_state(c)
    for i in range(n):
        c.append()
        if i % 7 == 0 or i == n - 1:
            full_check(c, c.random_q())
    check_state(c)


def test_decode_with_given_selection():
    c = _case(T0=1500, Bk=32, k=6)
    q = c.random_q()
    part = O.partition(c.T, c.S, c.W, c.Bk)
    for trial in range(4):
        sel = np.sort(c.rng.choice(part.nb, size=c.k, replace=False)).astype(np.int32)
        if trial == 3:
            sel[-2:] = -1
        out = c.decode_with_selection(q, sel.reshape(1, 1, -1))
        ref, _, _ = c.oracle_unit(q, 0, 0, sel=np.array([j for j in sel if j >= 0]))
        check_outputs(out[0], ref)
    assert c.layer.status(clear=True) == 0


def test_bad_selection_index_is_reported_and_skipped():
    from hybrid_sparse_linear_decode_b200 import HYB_STATUS_BAD_SELECTION
    c = _case(T0=1500, Bk=32, k=4)
    q = c.random_q()
    part = O.partition(c.T, c.S, c.W, c.Bk)
    sel = np.array([[[1, 5, part.nb + 3, 10 ** 6]]], dtype=np.int32)
    out = c.decode_with_selection(q, sel)
    assert c.layer.status(clear=True) & HYB_STATUS_BAD_SELECTION
    ref, _, _ = c.oracle_unit(q, 0, 0, sel=np.array([1, 5]))
    check_outputs(out[0], ref)
    assert c.layer.status() == 0


def test_ties_go_to_lower_block_index():
    """Blocks with identical keys have identical scores: the selection must
    take the lowest indices among them (exact on both sides)."""
    B, Hkv, d, S, W, Bk = 1, 1, 64, 4, 32, 16
    nbk = 20
    T0 = S + nbk * Bk + W
    rng = np.random.default_rng(3)
    Kf = rng.standard_normal((B, Hkv, T0, d))
    Vf = rng.standard_normal((B, Hkv, T0, d))
    blk = rng.standard_normal((Bk, d))
    for j in (2, 5, 9, 13, 17):            # five copies of one block
        Kf[0, 0, S + j * Bk:S + (j + 1) * Bk] = blk * 0.3 + 2.0
    from harness import bf16_bits
    c = Case(B, 4, Hkv, d, T0, Bk, S, W, 3, kv_bits=(bf16_bits(Kf), bf16_bits(Vf)))
    q = bf16_bits(np.abs(rng.standard_normal((1, 4, d))))
    out, sel, scores = c.decode(q)
    assert list(sel[0, 0]) == [2, 5, 9]
    s = scores[0, 0]
    assert s[2] == s[5] == s[9] == s[13] == s[17]


def test_step_host_matches_device_path():
    """The host-buffer entry point (copies + decode + append) equals the device path."""
    import torch
    c1 = _case(T0=1000, n_append=3, seed=5)
    c2 = _case(T0=1000, n_append=3, seed=5)
    for i in range(3):
        q = c1.random_q()
        c2.rng.standard_normal((c2.B, c2.Hq, c2.d))      # keep the rngs in step
        out1, _, _ = c1.decode(q, with_scores=False)
        c1.append()
        qh = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).pin_memory()
        kh = torch.from_numpy(np.ascontiguousarray(c2.Kb[:, :, c2.T]).view(np.int16)).view(torch.bfloat16).pin_memory()
        vh = torch.from_numpy(np.ascontiguousarray(c2.Vb[:, :, c2.T]).view(np.int16)).view(torch.bfloat16).pin_memory()
        oh = torch.empty((c2.B, c2.Hq, c2.d), dtype=torch.float32).pin_memory()
        c2.layer.step_host(qh, kh, vh, oh)
        torch.cuda.synchronize()
        c2.T += 1
        np.testing.assert_array_equal(oh.numpy(), out1.astype(np.float32))
    assert c1.layer.T == c2.layer.T


def test_step_layers_host_matches_device_path():
    """Several layers (different budgets) stepped from
    one host buffer with one copy in and one copy out equal the same layers
    stepped through the device entry point."""
    import torch
    import hybrid_sparse_linear_decode_b200 as H
    kws = [dict(T0=1000, W=64, k=4), dict(T0=1000, W=100, k=6), dict(T0=1000, W=32, k=2, Bk=16)]
    c1 = [_case(n_append=3, seed=30 + i, **kw) for i, kw in enumerate(kws)]
    c2 = [_case(n_append=3, seed=30 + i, **kw) for i, kw in enumerate(kws)]
    ctxs = [c.layer.ctx for c in c2]
    nbytes = H.hyb_attn_step_layers_staging_bytes(ctxs)
    staging = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    for step in range(3):
        qs = [c.random_q() for c in c1]
        for c, q in zip(c2, qs):
            c.rng.standard_normal((c.B, c.Hq, c.d))      # keep the rngs in step
        parts, ref = [], []
        for c, q in zip(c1, qs):
            out, _, _ = c.decode(q, with_scores=False)
            ref.append(out.astype(np.float32))
            parts += [q.reshape(-1), np.ascontiguousarray(c.Kb[:, :, c.T]).reshape(-1),
                      np.ascontiguousarray(c.Vb[:, :, c.T]).reshape(-1)]
            c.append()
        hin = torch.from_numpy(np.concatenate(parts).view(np.int16)).pin_memory()
        hout = torch.empty(sum(r.size for r in ref), dtype=torch.float32).pin_memory()
        H.hyb_attn_step_layers_host(ctxs, hin.data_ptr(), hout.data_ptr(), staging.data_ptr(), nbytes, stream)
        torch.cuda.synchronize()
        for c in c2:
            c.T += 1
        np.testing.assert_array_equal(hout.numpy(), np.concatenate([r.reshape(-1) for r in ref]))
    assert all(c.layer.T == c.T for c in c2)
    assert all(c.layer.status() == 0 for c in c2)


def test_capacity_error():
    import torch
    from hybrid_sparse_linear_decode_b200 import HybAttnError
    c = _case(T0=100, n_append=1)
    c.append()
    k = torch.zeros((1, 1, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(HybAttnError) as e:
        c.layer.append(k, k)
    assert e.value.code == -2


@pytest.mark.parametrize("kw,n", [
    (dict(T0=600, Bk=32, W=64), 70),                          # crosses block boundaries
    (dict(T0=200, W=0, Bk=8, k=3), 20),                       # W = 0: the appended token is evicted at once
    (dict(B=2, Hq=16, Hkv=4, T0=1500, Bk=64, W=100, k=5), 9),
])
def test_decode_append_equals_decode_then_append(kw, n):
    """The fused step (decode, then the token written by the selected-block
    kernel) gives the same outputs and selections as decode + append, and the
    final state and decode still match the oracle."""
    import torch
    c1 = _case(n_append=n, seed=11, **kw)
    c2 = _case(n_append=n, seed=11, **kw)
    dev = c1.layer.device
    from harness import to_device_bf16
    for i in range(n):
        q = c1.random_q()
        c2.rng.standard_normal((c2.B, c2.Hq, c2.d))      # keep the rngs in step
        out1, sel1, sc1 = c1.decode(q)
        c1.append()
        qd = to_device_bf16(q, dev)
        kd = to_device_bf16(np.ascontiguousarray(c2.Kb[:, :, c2.T]), dev)
        vd = to_device_bf16(np.ascontiguousarray(c2.Vb[:, :, c2.T]), dev)
        sel2 = torch.full((c2.B, c2.Hkv, c2.k), -7, dtype=torch.int32, device=dev)
        out2 = c2.layer.decode_append(qd, kd, vd, sel_out=sel2)
        torch.cuda.synchronize()
        c2.T += 1
        np.testing.assert_array_equal(out2.cpu().numpy(), out1.astype(np.float32))
        np.testing.assert_array_equal(sel2.cpu().numpy(), sel1)
    assert c1.layer.T == c2.layer.T == c2.T
    check_state(c2)
    full_check(c2, c2.random_q())
    assert c2.layer.status() == 0


def test_state_sync_is_idempotent_and_decode_folds():
    """After a decode nothing is pending (sync is a no-op); appends without a
    decode leave the state behind until a sync or the next decode folds them."""
    c = _case(T0=600, Bk=32, W=64, n_append=50)
    c.append(50)                         # 50 evictions pending
    full_check(c, c.random_q())          # the decode folds all of them
    s1 = c.state_gpu()
    s2 = c.state_gpu()
    for k in s1:
        np.testing.assert_array_equal(s1[k], s2[k])
    check_state(c)


@pytest.mark.parametrize("kw", [
    dict(T0=601, W=64, capacity=700, n_append=5),               # ragged last window piece
    dict(T0=4 + 64 + 32 * 5 + 7, capacity=400, n_append=3),     # newest block partial
    dict(T0=3, S=4, W=16, capacity=64, n_append=2),             # sinks only, one 4-row piece
    dict(B=2, Hq=16, Hkv=4, T0=1499, W=100, Bk=64, k=6, capacity=1600, n_append=4),
])
def test_unwritten_rows_past_T_do_not_leak(kw):
    """Cache rows at and past T are capacity nobody has written: here NaN.  A
    ragged chunk's last 16-row box reaches into them; with zero weights they
    must leave the result unchanged (0 * NaN would be NaN), before and after
    appends overwrite some of them."""
    c = _case(**kw)
    c.layer.k_cache[:, :, c.T:].fill_(float("nan"))
    c.layer.v_cache[:, :, c.T:].fill_(float("nan"))
    q = c.random_q()
    full_check(c, q)
    assert c.layer.status() == 0
    c.append(kw["n_append"])
    full_check(c, c.random_q())
    assert c.layer.status() == 0


@pytest.mark.parametrize("kw,n", [
    (dict(T0=600, n_append=64), 64),                                  # a block's worth, across a boundary
    (dict(T0=600, n_append=300, capacity=1000), 300),                 # one chunk evicts many blocks
    (dict(T0=40, S=4, W=64, n_append=50), 50),                        # the chunk starts the eviction
    (dict(B=2, Hq=16, Hkv=4, T0=1500, Bk=64, W=100, k=6, n_append=129), 129),
    (dict(d=64, T0=700, n_append=7), 7),
])
def test_append_chunk_matches_oracle(kw, n):
    """n tokens appended in one launch: the cache rows are the host's bits, and
    the next decode (which folds every token the chunk evicted) and the state
    match the oracle's definitions at the new length."""
    import torch
    from harness import to_device_bf16
    c = _case(**kw)
    dev = c.layer.device
    kb = to_device_bf16(np.ascontiguousarray(c.Kb[:, :, c.T:c.T + n]), dev)
    vb = to_device_bf16(np.ascontiguousarray(c.Vb[:, :, c.T:c.T + n]), dev)
    c.layer.append_chunk(kb, vb)
    c.T += n
    assert c.layer.T == c.T
    torch.cuda.synchronize()
    got = c.layer.k_cache[:, :, :c.T].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(got, c.Kb[:, :, :c.T].astype(np.uint16))
    full_check(c, c.random_q())
    assert c.layer.status() == 0
    check_state(c)


@pytest.mark.parametrize("kw,n", [
    (dict(T0=600, n_append=8), 8),                                    # two launches of 4 rows
    (dict(T0=4 + 64 + 32 * 5 - 3, n_append=6), 6),                   # 4 + 2 rows; the chunk completes a block
    (dict(B=2, Hq=16, Hkv=4, T0=1500, Bk=64, W=100, k=6, n_append=5), 5),   # 4 rows + 1
    (dict(T0=70, S=4, W=64, n_append=4), 4),                          # eviction starts inside the chunk
    (dict(T0=2, S=4, W=16, Bk=8, n_append=4), 4),                     # the sinks fill inside the chunk
    (dict(T0=300, S=3, W=20, Bk=1, k=12, n_append=4), 4),             # one-token blocks: E tokens in 3 blocks
    (dict(Hq=8, Hkv=8, d=64, T0=900, Bk=16, W=40, k=5, n_append=2), 2),     # G = 1, 2 rows
    (dict(B=2, Hq=8, Hkv=2, T0=4 + 64 + 8 * 1300, Bk=8, W=64, k=20, n_append=2), 2),  # 1300 blocks, 2 rows
    (dict(B=4, Hq=32, Hkv=8, T0=5000, Bk=64, W=1024, k=16, n_append=4), 4),  # 32 units
])
def test_decode_chunk_rows_match_oracle(kw, n):
    """Speculative verification of n draft tokens: row j is the decode at length
    T + j (the chunk's tokens before j included), against the oracle at that
    length; the state after the chunk against the oracle at T + n."""
    import torch
    from harness import to_device_bf16
    c = _case(**kw)
    dev = c.layer.device
    qs = np.stack([c.random_q() for _ in range(n)])
    q = to_device_bf16(qs, dev)
    kb = to_device_bf16(np.ascontiguousarray(c.Kb[:, :, c.T:c.T + n].transpose(2, 0, 1, 3)), dev)
    vb = to_device_bf16(np.ascontiguousarray(c.Vb[:, :, c.T:c.T + n].transpose(2, 0, 1, 3)), dev)
    sel = torch.full((n, c.B, c.Hkv, c.k), -7, dtype=torch.int32, device=dev)
    out = c.layer.decode_chunk(q, kb, vb, sel_out=sel)
    torch.cuda.synchronize()
    out, sel = out.cpu().numpy().astype(np.float64), sel.cpu().numpy()
    T0 = c.T
    for j in range(n):
        c.T = T0 + j
        refs, gots = [], []
        for b in range(c.B):
            for h in range(c.Hkv):
                _, _, oscores = c.oracle_unit(qs[j], b, h)
                check_selection(sel[j, b, h], oscores, c.k)
                gsel = np.array([int(x) for x in sel[j, b, h] if x >= 0], dtype=np.int64)
                ref, _, _ = c.oracle_unit(qs[j], b, h, sel=gsel)
                refs.append(ref)
                gots.append(out[j, b, h * c.G:(h + 1) * c.G])
        check_outputs(np.array(gots), np.array(refs))
    c.T = T0 + n
    assert c.layer.T == c.T and c.layer.status() == 0
    check_state(c)


@pytest.mark.parametrize("nbk,copies,k,d", [
    (700, (3, 150, 333, 480, 690), 3, 64),    # one unit: a cluster of 16 ranks, copies in different shares
    (1300, (10, 11, 700, 1299), 2, 128),      # the second copy in the same share, the last in the last share
])
def test_ties_across_rank_shares_above_512_blocks(nbk, copies, k, d):
    """Above 512 blocks (the selection's multi-pass path, its bound from the
    lanes' two largest keys): blocks with identical scores, in different ranks'
    shares of the scoring, must still go to the lowest indices."""
    B, Hkv, S, W, Bk = 1, 1, 4, 32, 8
    T0 = S + nbk * Bk + W
    rng = np.random.default_rng(5)
    Kf = rng.standard_normal((B, Hkv, T0, d))
    Vf = rng.standard_normal((B, Hkv, T0, d))
    blk = rng.standard_normal((Bk, d))
    for j in copies:
        Kf[0, 0, S + j * Bk:S + (j + 1) * Bk] = blk * 0.3 + 2.0
    from harness import bf16_bits
    c = Case(B, 4, Hkv, d, T0, Bk, S, W, k, kv_bits=(bf16_bits(Kf), bf16_bits(Vf)))
    q = bf16_bits(np.abs(rng.standard_normal((1, 4, d))))
    out, sel, scores = c.decode(q)
    assert list(sel[0, 0]) == sorted(copies)[:k]
    s = scores[0, 0]
    assert all(s[j] == s[copies[0]] for j in copies)
    full_check(c, q)


@pytest.mark.parametrize("kw", [
    dict(T0=4 + 64 + 8 * 900, Bk=8, W=64, k=20),                       # one unit, 900 blocks
    dict(B=2, Hq=8, Hkv=2, T0=4 + 128 + 16 * 600, Bk=16, W=128, k=32),  # 4 units, k = 32
    dict(d=64, T0=4 + 64 + 8 * 800, Bk=8, W=64, k=12),                 # head dim 64
])
def test_selection_above_512_blocks(kw):
    c = _case(**kw)
    full_check(c, c.random_q())
    assert c.layer.status() == 0


def test_distributed_selection_with_all_scores_equal():
    """Above 512 blocks each rank selects its own share's top-k and the ranks
    merge their candidates.  With q = 0 every score is 0: the k lowest block
    indices must be selected (ties to the lower index, across ranks), the share
    of a rank holds more equal keys than its gather segments (the radix
    fallback inside the rank), and the output is the mean of V."""
    import torch
    c = _case(B=16, Hq=16, Hkv=4, d=64, T0=4 + 16 + 8 * 1100, Bk=8, S=4, W=16, k=16, seed=13)
    q = np.zeros((c.B, c.Hq, c.d), dtype=np.uint16)
    out, sel, _ = c.decode(q)
    assert (sel == np.arange(16, dtype=np.int32)[None, None, :]).all()
    for b, h in ((0, 0), (15, 3), (7, 2)):
        Kf, Vf = c.unit_kv(b, h)
        check_outputs(out[b, h * c.G:(h + 1) * c.G], np.broadcast_to(Vf.mean(axis=0), (c.G, c.d)),
                      max_abs=1e-4, rel_l2=1e-4)
    assert c.layer.status() == 0


@pytest.mark.parametrize("kw", [
    dict(T0=600, Bk=1, S=4, W=32, k=16),                        # 564 one-token blocks: the distributed selection
    dict(T0=600, Bk=1, S=4, W=32, k=40),                        # k > 32: the radix selection
    dict(B=2, Hq=8, Hkv=2, d=64, T0=300, Bk=1, S=2, W=20, k=12),
])
def test_token_granular_exact_set(kw):
    """Token granularity (the block size 1): the exact set is the sinks, the
    window and the top-k evicted tokens by their group-summed score s_t; every
    other evicted token takes the Taylor weight through the subtraction form."""
    c = _case(**kw)
    full_check(c, c.random_q())
    c2 = _case(n_append=5, **kw)
    c2.append(5)
    full_check(c2, c2.random_q())
    check_state(c2)
    assert c.layer.status() == 0 and c2.layer.status() == 0


def test_decode_chunk_repeated_chunks_and_state():
    """Speculative verification, chunk after chunk (each call folds the
    evictions the previous chunk left pending): 5 chunks of 4 draft rows, every
    row against the oracle at its own length, then the state."""
    import torch
    from harness import to_device_bf16
    c = _case(B=2, Hq=16, Hkv=4, T0=1200, Bk=32, W=64, k=6, n_append=20, seed=17)
    dev = c.layer.device
    n = 4
    for step in range(5):
        qs = np.stack([c.random_q() for _ in range(n)])
        kb = to_device_bf16(np.ascontiguousarray(c.Kb[:, :, c.T:c.T + n].transpose(2, 0, 1, 3)), dev)
        vb = to_device_bf16(np.ascontiguousarray(c.Vb[:, :, c.T:c.T + n].transpose(2, 0, 1, 3)), dev)
        sel = torch.full((n, c.B, c.Hkv, c.k), -7, dtype=torch.int32, device=dev)
        out = c.layer.decode_chunk(to_device_bf16(qs, dev), kb, vb, sel_out=sel)
        torch.cuda.synchronize()
        out, sel = out.cpu().numpy().astype(np.float64), sel.cpu().numpy()
        T0 = c.T
        for j in range(n):
            c.T = T0 + j
            refs, gots = [], []
            for b in range(c.B):
                for h in range(c.Hkv):
                    _, _, oscores = c.oracle_unit(qs[j], b, h)
                    check_selection(sel[j, b, h], oscores, c.k)
                    gsel = np.array([int(x) for x in sel[j, b, h] if x >= 0], dtype=np.int64)
                    ref, _, _ = c.oracle_unit(qs[j], b, h, sel=gsel)
                    refs.append(ref)
                    gots.append(out[j, b, h * c.G:(h + 1) * c.G])
            check_outputs(np.array(gots), np.array(refs))
        c.T = T0 + n
    assert c.layer.T == c.T and c.layer.status() == 0
    check_state(c)
    full_check(c, c.random_q())
