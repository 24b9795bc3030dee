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
