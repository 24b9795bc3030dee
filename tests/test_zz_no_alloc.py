"""The no-allocation decode entry point against the regular one.

Some callers cannot allocate device memory themselves (they run under an
allocator they do not own, or must not call cudaMalloc/cudaFree on their hot
path).  hyb_attn_decode_noalloc serves them from a fixed device array inside the
library; its results must equal those of hyb_attn_decode, call after call.
This file is collected last so that a failure here stops a run only after every
other test has run.
"""

import numpy as np
import pytest

from harness import Case, OUT_MAX_ABS, OUT_REL_L2, check_outputs, to_device_bf16

pytestmark = pytest.mark.gpu


def test_decode_noalloc_matches_decode_twice():
    import torch
    import hybrid_sparse_linear_decode_b200 as H
    c = Case(B=2, Hq=16, Hkv=4, d=128, T0=3000, Bk=64, S=4, W=256, k=8, n_append=2, seed=11)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        q = to_device_bf16(c.random_q(), c.layer.device)
        sel_ref = torch.full((c.B, c.Hkv, c.k), -7, dtype=torch.int32, device=c.layer.device)
        ref = c.layer.decode(q, sel_out=sel_ref)
        out = torch.full_like(ref, float("nan"))
        sel = torch.full_like(sel_ref, -7)
        H.hyb_attn_decode_noalloc(c.layer.ctx, q.data_ptr(), out.data_ptr(), sel.data_ptr(), stream)
        torch.cuda.synchronize()
        assert torch.equal(sel, sel_ref)
        check_outputs(out.cpu().numpy().astype(np.float64), ref.cpu().numpy().astype(np.float64),
                      max_abs=OUT_MAX_ABS, rel_l2=OUT_REL_L2)
        # the call's device status bits land in the context's status word
        assert c.layer.status() == 0
        c.append()   # the second call sees a longer history
