"""The CUDA twin of the input generator produces the same bits as the numpy
generator (so device-filled caches and host-regenerated oracle inputs agree)."""

import numpy as np
import pytest

from syngen import configs as C
from syngen import host as SH

pytestmark = pytest.mark.gpu


def test_normals_bit_identical():
    import syngen.device as SD
    SD.build()
    key = SH.stream_key(0, C.STREAM_K)
    for idx0 in (0, 123_456_789, 2 ** 40 + 17):
        dev = SD.normal(key, idx0, 1 << 16, "cuda").cpu().numpy()
        host = SH.normal(key, np.arange(idx0, idx0 + (1 << 16), dtype=np.uint64))
        assert np.array_equal(dev.view(np.uint64), host.view(np.uint64))


@pytest.mark.parametrize("name,layer", [("tiny", 0), ("llama8b_32k_layer", 0), ("llama8b_32layers_b8_32k", 7),
                                        ("llama8b_32layers_b4_128k", 3), ("llama8b_256k_256steps", 0)])
def test_kv_slices_bit_identical(name, layer):
    import torch
    import syngen.device as SD
    SD.build()
    w = C.get_workload(name)
    tb = SD.DeviceTables(w, layer, "cuda")
    t0, t1 = 0, min(w.T0, 3000)
    shp = (w.batch, w.n_kv_heads, t1 - t0, w.head_dim)
    k = torch.empty(shp, dtype=torch.bfloat16, device="cuda")
    v = torch.empty(shp, dtype=torch.bfloat16, device="cuda")
    SD.fill_kv(w, tb, k, v, t0, t1, t_out0=t0)
    # a late slice too (planted / offset blocks live anywhere in [S, T0 - W))
    t2, t3 = w.T0 - 700, w.T0 + 5
    shp2 = (w.batch, w.n_kv_heads, t3 - t2, w.head_dim)
    k2 = torch.empty(shp2, dtype=torch.bfloat16, device="cuda")
    v2 = torch.empty(shp2, dtype=torch.bfloat16, device="cuda")
    SD.fill_kv(w, tb, k2, v2, t2, t3, t_out0=t2)
    kk = k.view(torch.int16).cpu().numpy().view(np.uint16)
    vv = v.view(torch.int16).cpu().numpy().view(np.uint16)
    kk2 = k2.view(torch.int16).cpu().numpy().view(np.uint16)
    vv2 = v2.view(torch.int16).cpu().numpy().view(np.uint16)
    for b, h in [(0, 0), (w.batch - 1, w.n_kv_heads - 1)]:
        hk, hv = SH.kv_bits(w, tb.host, b, h, t0, t1)
        assert np.array_equal(kk[b, h], hk) and np.array_equal(vv[b, h], hv)
        hk2, hv2 = SH.kv_bits(w, tb.host, b, h, t2, t3)
        assert np.array_equal(kk2[b, h], hk2) and np.array_equal(vv2[b, h], hv2)
    if w.n_planted:
        # planted blocks reproduce too
        for j in tb.host.planted[0, 0][:2]:
            a = w.n_sink + int(j) * w.block_size
            kd = torch.empty((w.batch, w.n_kv_heads, w.block_size, w.head_dim), dtype=torch.bfloat16, device="cuda")
            vd = torch.empty_like(kd)
            SD.fill_kv(w, tb, kd, vd, a, a + w.block_size, t_out0=a)
            hk, _ = SH.kv_bits(w, tb.host, 0, 0, a, a + w.block_size)
            assert np.array_equal(kd.view(torch.int16).cpu().numpy().view(np.uint16)[0, 0], hk)
