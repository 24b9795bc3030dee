"""Strided block selection (one reading of the SPLA table-of-contents heading
"Strided block selection", whose body the page does not give): the last block
of every `stride` candidate blocks always exact, plus the top-k of the others.
The CUDA path (a selection launch, then the decode with that selection) against
the fp64 oracle unit by unit: the strided blocks exactly, the top-k part with
the harness's tie window, and the outputs given the GPU's selection."""

import numpy as np
import pytest

import oracle as O
from harness import SEL_TIE, Case, bits_to_f64, check_outputs

pytestmark = pytest.mark.gpu


def _check(case, q_bits, k_top, stride, appends=0):
    import torch
    from harness import to_device_bf16
    for _ in range(appends):
        case.append()
    dev = case.layer.device
    q = to_device_bf16(q_bits, dev)
    sel = torch.full((case.B, case.Hkv, case.k), -7, dtype=torch.int32, device=dev)
    out = case.layer.decode_strided(q, k_top, stride, sel_out=sel)
    torch.cuda.synchronize()
    out, sel = out.cpu().numpy().astype(np.float64), sel.cpu().numpy()
    assert case.layer.status() == 0
    refs, gots = [], []
    for b in range(case.B):
        for h in range(case.Hkv):
            K, V = case.unit_kv(b, h)
            part = O.partition(case.T, case.S, case.W, case.Bk)
            qf = bits_to_f64(q_bits)[b, h * case.G:(h + 1) * case.G]
            mu, var = O.block_stats(K, part)
            scores = O.block_scores(qf, mu, var, case.scale) if part.nb else np.zeros(0)
            want = O.select_blocks_strided(scores, k_top, stride)
            row = [int(j) for j in sel[b, h]]
            n = len(want)
            assert all(j == -1 for j in row[n:]), row
            got = row[:n]
            assert got == sorted(got) and len(set(got)) == n, got
            fixed = set(int(j) for j in O.strided_blocks(part.nb, stride))
            assert fixed <= set(got), (sorted(fixed - set(got)), got)
            # the top-k part: any difference must be a tie at the k-th score
            diff = set(got) ^ set(int(j) for j in want)
            if diff:
                others = np.array([scores[j] for j in range(part.nb) if j not in fixed])
                kth = np.sort(others)[::-1][min(k_top, others.size) - 1]
                for j in diff:
                    assert abs(scores[j] - kth) <= SEL_TIE * max(1.0, abs(kth)), (j, scores[j], kth)
            refs.append(O.hybrid_subtract(qf, K, V, part, np.array(got, dtype=np.int64), case.scale))
            gots.append(out[b, h * case.G:(h + 1) * case.G])
    check_outputs(np.array(gots), np.array(refs))


@pytest.mark.parametrize("k_top,stride", [(4, 8), (0, 3), (6, 1000), (2, 1)])
def test_strided_selection_matches_oracle(k_top, stride):
    """Ragged last block (T0 - S - W not a multiple of Bk), several units, a
    stride past the block count (plain top-k), stride 1 (every block: full
    softmax), no top-k at all."""
    nb = (2500 - 4 - 100 + 31) // 32
    width = nb // stride + min(k_top, nb - nb // stride)
    c = Case(B=2, Hq=8, Hkv=2, d=128, T0=2500, Bk=32, S=4, W=100, k=max(width, 1), n_append=3, seed=31)
    _check(c, c.random_q(), k_top, stride)


def test_strided_selection_after_appends_and_d64():
    """Pending evictions folded before the scores (the selection launch reads
    the statistics), head dimension 64, group of 2."""
    nb_after = (1500 + 5 - 4 - 64 + 15) // 16
    c = Case(B=1, Hq=4, Hkv=2, d=64, T0=1500, Bk=16, S=4, W=64, k=nb_after // 4 + 5, n_append=5, seed=32)
    _check(c, c.random_q(), 5, 4, appends=5)


def test_strided_selection_arguments_are_checked():
    from hybrid_sparse_linear_decode_b200 import HybAttnError
    import torch
    from harness import to_device_bf16
    c = Case(B=1, Hq=4, Hkv=1, d=64, T0=800, Bk=16, S=4, W=64, k=8, seed=33)
    q = to_device_bf16(c.random_q(), c.layer.device)
    for k_top, stride in ((4, 0), (-1, 4), (8, 2)):  # stride 0, negative k, union wider than top_k
        with pytest.raises(HybAttnError):
            c.layer.decode_strided(q, k_top, stride)
    torch.cuda.synchronize()


@pytest.mark.parametrize("nbk,k_top,stride,d", [
    (300, 40, 5, 128),    # k above 32: the selection by rounds of block-wide maxima
    (700, 16, 50, 128),   # 686 non-strided blocks: the one-warp selection above 512 scores
    (520, 32, 3, 64),     # k = 32, head dimension 64, 347 candidates
])
def test_strided_selection_wide_k_and_many_blocks(nbk, k_top, stride, d):
    S, W, Bk = 4, 64, 8
    T0 = S + nbk * Bk + W + 5  # a ragged last block
    nb = (T0 - S - W + Bk - 1) // Bk
    width = nb // stride + min(k_top, nb - nb // stride)
    c = Case(B=1, Hq=4, Hkv=1, d=d, T0=T0, Bk=Bk, S=S, W=W, k=width, seed=34)
    _check(c, c.random_q(), k_top, stride)


@pytest.mark.parametrize("nbk,k_top,stride", [
    (600, 10, 7),   # 515 candidates tie: more than the one-warp selection ranks, above 512
    (400, 24, 9),   # 356 candidates tie, below 512
])
def test_strided_selection_all_scores_equal(nbk, k_top, stride):
    """q = 0 makes every score 0: the strided blocks and the k lowest other
    block indices, exactly; every token weighs 1, so the output is the mean of V."""
    import torch
    from harness import to_device_bf16
    S, W, Bk = 4, 16, 8
    nb = nbk
    width = nb // stride + k_top
    c = Case(B=2, Hq=4, Hkv=2, d=64, T0=S + nbk * Bk + W, Bk=Bk, S=S, W=W, k=width, seed=35)
    dev = c.layer.device
    q = to_device_bf16(np.zeros((c.B, c.Hq, c.d), dtype=np.uint16), dev)
    sel = torch.full((c.B, c.Hkv, c.k), -7, dtype=torch.int32, device=dev)
    out = c.layer.decode_strided(q, k_top, stride, sel_out=sel)
    torch.cuda.synchronize()
    out, sel = out.cpu().numpy().astype(np.float64), sel.cpu().numpy()
    assert c.layer.status() == 0
    fixed = [j for j in range(nb) if j % stride == stride - 1]
    others = [j for j in range(nb) if j % stride != stride - 1]
    want = sorted(fixed + others[:k_top])
    for b in range(c.B):
        for h in range(c.Hkv):
            assert list(sel[b, h]) == want
            _, Vf = c.unit_kv(b, h)
            check_outputs(out[b, h * c.G:(h + 1) * c.G], np.broadcast_to(Vf.mean(axis=0), (c.G, c.d)),
                          max_abs=1e-4, rel_l2=1e-4)


@pytest.mark.parametrize("appends,Bk,d", [(1, 16, 128), (3, 4, 64), (4, 4, 128), (2, 1, 64)])
def test_strided_selection_folds_pending_evictions(appends, Bk, d):
    """One to four appends since the last fold (a decode step's usual case):
    the selection launch scores the blocks that hold them from rows folded on
    the fly, and the decode folds them into the state.  The first pending token
    is the last of its block, so the ones after it open a new block (with
    blocks of one token, every pending token is a block of its own)."""
    from harness import check_state
    S, W, nblk = 4, 64, 300
    T0 = S + W + nblk * Bk + (Bk - 1)
    nb = (T0 + appends - W - S + Bk - 1) // Bk
    k_top, stride = 6, 5
    c = Case(B=1, Hq=4, Hkv=2, d=d, T0=T0, Bk=Bk, S=S, W=W, k=nb // stride + k_top, n_append=appends, seed=36)
    _check(c, c.random_q(), k_top, stride, appends=appends)
    assert c.layer.status() == 0
    check_state(c)
