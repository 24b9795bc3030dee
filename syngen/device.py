"""CUDA twin of the generator (``libsyngen.so``): fills device KV caches.

Builds with ``syngen.device.build()`` (nvcc, sm_100a).  The caller passes torch
CUDA tensors; tables (planted blocks, q_hat, head scales) are computed on the
host by ``syngen.host`` and copied to the device here.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from . import configs as C
from . import host as H

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "libsyngen.so")
SRC = os.path.join(HERE, "csrc", "syngen.cu")


def _nvcc() -> str:
    return os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = [_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-o", LIB + ".tmp", SRC]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise RuntimeError(f"{LIB} is missing: run syngen.device.build()")
        lib = ctypes.CDLL(LIB)
        i32, i64, u64, vp, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_void_p, ctypes.c_double
        lib.syngen_fill_kv.restype = ctypes.c_int
        lib.syngen_fill_kv.argtypes = [vp, vp, i64, i64, i64, i64, u64, u64, u64, i32, i32, i32, i32, i32, i32,
                                       i64, vp, i32, vp, f64, f64, f64, vp, i64, i64, vp]
        lib.syngen_normal.restype = ctypes.c_int
        lib.syngen_normal.argtypes = [vp, u64, u64, i64, vp]
        _lib = lib
    return _lib


class DeviceTables:
    """Per-layer host tables copied to the device once."""

    def __init__(self, w: C.Workload, layer: int, device):
        import torch
        t = H.LayerTables(w, layer)
        self.host = t
        self.planted = torch.from_numpy(np.ascontiguousarray(t.planted, dtype=np.int32)).to(device)
        self.qhat = torch.from_numpy(np.ascontiguousarray(t.qhat, dtype=np.float64)).to(device)
        self.scale = torch.from_numpy(np.ascontiguousarray(t.scale, dtype=np.float64)).to(device)


def fill_kv(w: C.Workload, tables: DeviceTables, k, v, t_begin: int, t_end: int, t_out0: int = 0, stream=None):
    """Write positions [t_begin, t_end) of every (b, kv head) of the layer into
    ``k``/``v`` (torch bf16 CUDA tensors [B][Hkv][rows][d]; row r = position
    t_out0 + r)."""
    import torch
    lib = _load()
    assert k.dtype == torch.bfloat16 and k.is_cuda and k.is_contiguous() and v.is_contiguous()
    B, Hkv, rows, d = k.shape
    assert (B, Hkv, d) == (w.batch, w.n_kv_heads, w.head_dim)
    assert t_out0 <= t_begin and t_end - t_out0 <= rows
    s = stream if stream is not None else torch.cuda.current_stream().cuda_stream
    rc = lib.syngen_fill_kv(
        k.data_ptr(), v.data_ptr(), rows, t_begin, t_end, t_out0,
        H.stream_key(w.seed, C.STREAM_K), H.stream_key(w.seed, C.STREAM_V),
        H.stream_key(w.seed, C.STREAM_BLOCK_OFFSET), tables.host.layer, w.batch, w.n_kv_heads, w.head_dim,
        w.n_sink, w.block_size, w.n_sink + w.evicted(w.T0), tables.planted.data_ptr() if w.n_planted else None,
        w.n_planted, tables.qhat.data_ptr(), w.planted_amp, w.planted_std, w.block_offset_std,
        tables.scale.data_ptr(), C.TOKEN_STRIDE, C.BLOCK_STRIDE, s)
    if rc != 0:
        raise RuntimeError(f"syngen_fill_kv failed with CUDA error {rc}")


def normal(key: int, idx0: int, n: int, device):
    import torch
    lib = _load()
    out = torch.empty(n, dtype=torch.float64, device=device)
    rc = lib.syngen_normal(out.data_ptr(), key, idx0, n, torch.cuda.current_stream().cuda_stream)
    if rc != 0:
        raise RuntimeError(f"syngen_normal failed with CUDA error {rc}")
    return out
