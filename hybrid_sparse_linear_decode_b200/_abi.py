"""ctypes binding of ``include/hyb_attn.h``: argument marshalling only.

Every function here has the name of the C entry point it calls and raises
``HybAttnError`` on a negative return code.  Pointers are plain integers
(``tensor.data_ptr()``) and streams are ``cudaStream_t`` handles as integers
(``torch.cuda.Stream.cuda_stream``).  Nothing is computed in Python: a missing
library is an error, there is no fallback.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libhyb_attn.so")

HYB_OK = 0
HYB_EINVAL = -1
HYB_ECAPACITY = -2
HYB_ECUDA = -3
HYB_ESTATE = -4
HYB_ENOMEM = -5
HYB_ESCRATCH = -6

HYB_STATUS_NONFINITE = 0x1
HYB_STATUS_DENOMINATOR = 0x2
HYB_STATUS_BAD_SELECTION = 0x4
HYB_STATUS_TIMEOUT = 0x8
HYB_STATUS_NAN_SCORE = 0x10

HYB_TEST_WITHHOLD_SCORES = 0x1

c_i32, c_i64, c_f32, c_vp, c_sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t


class hyb_attn_config(ctypes.Structure):
    _fields_ = [("batch", c_i32), ("n_q_heads", c_i32), ("n_kv_heads", c_i32), ("head_dim", c_i32),
                ("block_size", c_i32), ("n_sink", c_i32), ("window", c_i32), ("top_k", c_i32),
                ("capacity", c_i64), ("scale", c_f32),
                ("head_window", ctypes.POINTER(c_i32)), ("head_top_k", ctypes.POINTER(c_i32))]


class hyb_attn_sizes(ctypes.Structure):
    _fields_ = [("kv_cache_elems", c_i64), ("H_elems", c_i64), ("z_elems", c_i64), ("n_elems", c_i64),
                ("max_blocks", c_i64), ("stats_elems", c_i64), ("workspace_bytes", c_i64)]


class hyb_attn_buffers(ctypes.Structure):
    _fields_ = [("k_cache", c_vp), ("v_cache", c_vp), ("H", c_vp), ("zk", c_vp), ("zv", c_vp), ("n", c_vp),
                ("mu", c_vp), ("var", c_vp), ("workspace", c_vp), ("workspace_bytes", c_sz)]


class hyb_attn_plan_info(ctypes.Structure):
    _fields_ = [("T", c_i64), ("n_blocks", c_i64), ("k_eff", c_i64), ("exact_tokens", c_i64),
                ("chunks_per_unit", c_i32), ("cluster_ctas", c_i32), ("grid_ctas", c_i32)]


# (name, restype, argtypes) of every entry point declared in include/hyb_attn.h
SIGNATURES = [
    ("hyb_attn_query_sizes", ctypes.c_int, [ctypes.POINTER(hyb_attn_config), ctypes.POINTER(hyb_attn_sizes)]),
    ("hyb_attn_workspace_size", c_sz, [ctypes.POINTER(hyb_attn_config)]),
    ("hyb_attn_plan", ctypes.c_int, [ctypes.POINTER(hyb_attn_config), c_i64, c_i32,
                                     ctypes.POINTER(hyb_attn_plan_info)]),
    ("hyb_attn_init", ctypes.c_int, [ctypes.POINTER(c_vp), ctypes.POINTER(hyb_attn_config),
                                     ctypes.POINTER(hyb_attn_buffers), c_i64, c_vp]),
    ("hyb_attn_init_rows", ctypes.c_int, [ctypes.POINTER(c_vp), ctypes.POINTER(hyb_attn_config),
                                          ctypes.POINTER(hyb_attn_buffers), ctypes.POINTER(c_i64), c_vp]),
    ("hyb_attn_attach", ctypes.c_int, [ctypes.POINTER(c_vp), ctypes.POINTER(hyb_attn_config),
                                       ctypes.POINTER(hyb_attn_buffers), c_i64, c_vp]),
    ("hyb_attn_attach_rows", ctypes.c_int, [ctypes.POINTER(c_vp), ctypes.POINTER(hyb_attn_config),
                                            ctypes.POINTER(hyb_attn_buffers), ctypes.POINTER(c_i64), c_vp]),
    ("hyb_attn_append", ctypes.c_int, [c_vp, c_vp, c_vp, c_vp]),
    ("hyb_attn_append_chunk", ctypes.c_int, [c_vp, c_vp, c_vp, c_i32, c_vp]),
    ("hyb_attn_sync_state", ctypes.c_int, [c_vp, c_vp]),
    ("hyb_attn_decode", ctypes.c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]),
    ("hyb_attn_decode_append", ctypes.c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]),
    ("hyb_attn_decode_chunk", ctypes.c_int, [c_vp, c_vp, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp]),
    ("hyb_attn_decode_with_selection", ctypes.c_int, [c_vp, c_vp, c_vp, c_vp, c_vp]),
    ("hyb_attn_decode_strided", ctypes.c_int, [c_vp, c_vp, c_i32, c_i32, c_vp, c_vp, c_vp]),
    ("hyb_attn_step_host", ctypes.c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]),
    ("hyb_attn_step_layers_staging_bytes", c_sz, [ctypes.POINTER(c_vp), c_i32]),
    ("hyb_attn_step_layers_host", ctypes.c_int, [ctypes.POINTER(c_vp), c_i32, c_vp, c_vp, c_vp, c_sz, c_vp]),
    ("hyb_attn_decode_noalloc", ctypes.c_int, [c_vp, c_vp, c_vp, c_vp, c_vp]),
    ("hyb_attn_length", c_i64, [c_vp]),
    ("hyb_attn_row_length", c_i64, [c_vp, c_i32]),
    ("hyb_attn_status", ctypes.c_int, [c_vp, ctypes.POINTER(ctypes.c_uint32), ctypes.c_int, c_vp]),
    ("hyb_attn_set_timing_events", ctypes.c_int, [c_vp, c_vp, c_vp]),
    ("hyb_attn_set_wait_limit", ctypes.c_int, [c_vp, ctypes.c_uint64]),
    ("hyb_attn_set_test_flags", ctypes.c_int, [c_vp, ctypes.c_uint32]),
    ("hyb_attn_destroy", None, [c_vp]),
    ("hyb_attn_strerror", ctypes.c_char_p, [ctypes.c_int]),
    ("hyb_attn_last_cuda_error", ctypes.c_char_p, []),
]


class HybAttnError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        msg = f"{fn} failed: {code} ({strerror(code)})"
        if code == HYB_ECUDA:
            msg += f" [{hyb_attn_last_cuda_error()}]"
        super().__init__(msg)


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load ``libhyb_attn.so`` (built by ``hybrid_sparse_linear_decode_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"{path} not found: build it with `python -m hybrid_sparse_linear_decode_b200.build`")
        lib = ctypes.CDLL(path)
        for name, res, args in SIGNATURES:
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def _check(fn: str, rc: int) -> int:
    if rc < 0:
        raise HybAttnError(fn, rc)
    return rc


def strerror(code: int) -> str:
    return load_library().hyb_attn_strerror(code).decode()


hyb_attn_strerror = strerror


def hyb_attn_last_cuda_error() -> str:
    return load_library().hyb_attn_last_cuda_error().decode()


def hyb_attn_query_sizes(cfg: hyb_attn_config) -> hyb_attn_sizes:
    out = hyb_attn_sizes()
    _check("hyb_attn_query_sizes", load_library().hyb_attn_query_sizes(ctypes.byref(cfg), ctypes.byref(out)))
    return out


def hyb_attn_workspace_size(cfg: hyb_attn_config) -> int:
    return int(load_library().hyb_attn_workspace_size(ctypes.byref(cfg)))


def hyb_attn_plan(cfg: hyb_attn_config, T: int, n_sm: int) -> hyb_attn_plan_info:
    out = hyb_attn_plan_info()
    _check("hyb_attn_plan", load_library().hyb_attn_plan(ctypes.byref(cfg), T, n_sm, ctypes.byref(out)))
    return out


def hyb_attn_init(cfg: hyb_attn_config, buf: hyb_attn_buffers, T0: int, stream: int) -> int:
    h = c_vp()
    _check("hyb_attn_init", load_library().hyb_attn_init(ctypes.byref(h), ctypes.byref(cfg), ctypes.byref(buf),
                                                         T0, stream))
    return h.value


def _i64_array(vals):
    return (c_i64 * len(vals))(*[int(v) for v in vals])


def hyb_attn_init_rows(cfg: hyb_attn_config, buf: hyb_attn_buffers, row_T0, stream: int) -> int:
    h = c_vp()
    _check("hyb_attn_init_rows", load_library().hyb_attn_init_rows(ctypes.byref(h), ctypes.byref(cfg),
                                                                   ctypes.byref(buf), _i64_array(row_T0), stream))
    return h.value


def hyb_attn_attach_rows(cfg: hyb_attn_config, buf: hyb_attn_buffers, row_T, stream: int) -> int:
    h = c_vp()
    _check("hyb_attn_attach_rows", load_library().hyb_attn_attach_rows(ctypes.byref(h), ctypes.byref(cfg),
                                                                       ctypes.byref(buf), _i64_array(row_T),
                                                                       stream))
    return h.value


def hyb_attn_attach(cfg: hyb_attn_config, buf: hyb_attn_buffers, T: int, stream: int) -> int:
    h = c_vp()
    _check("hyb_attn_attach", load_library().hyb_attn_attach(ctypes.byref(h), ctypes.byref(cfg), ctypes.byref(buf),
                                                             T, stream))
    return h.value


def hyb_attn_append(ctx: int, k_new: int, v_new: int, stream: int) -> None:
    _check("hyb_attn_append", load_library().hyb_attn_append(ctx, k_new, v_new, stream))


def hyb_attn_append_chunk(ctx: int, k_new: int, v_new: int, n: int, stream: int) -> None:
    _check("hyb_attn_append_chunk", load_library().hyb_attn_append_chunk(ctx, k_new, v_new, n, stream))


def hyb_attn_sync_state(ctx: int, stream: int) -> None:
    _check("hyb_attn_sync_state", load_library().hyb_attn_sync_state(ctx, stream))


def hyb_attn_decode(ctx: int, q: int, out: int, sel_out, scores_out, stream: int) -> None:
    _check("hyb_attn_decode", load_library().hyb_attn_decode(ctx, q, out, sel_out, scores_out, stream))


def hyb_attn_decode_append(ctx: int, q: int, k_new: int, v_new: int, out: int, sel_out, scores_out,
                           stream: int) -> None:
    _check("hyb_attn_decode_append",
           load_library().hyb_attn_decode_append(ctx, q, k_new, v_new, out, sel_out, scores_out, stream))


def hyb_attn_decode_chunk(ctx: int, q: int, k_new: int, v_new: int, n: int, out: int, sel_out,
                          stream: int) -> None:
    _check("hyb_attn_decode_chunk",
           load_library().hyb_attn_decode_chunk(ctx, q, k_new, v_new, n, out, sel_out, stream))


def hyb_attn_decode_with_selection(ctx: int, q: int, sel: int, out: int, stream: int) -> None:
    _check("hyb_attn_decode_with_selection",
           load_library().hyb_attn_decode_with_selection(ctx, q, sel, out, stream))


def hyb_attn_decode_strided(ctx: int, q: int, k_top: int, stride: int, out: int, sel_out: int, stream: int) -> None:
    _check("hyb_attn_decode_strided",
           load_library().hyb_attn_decode_strided(ctx, q, k_top, stride, out, sel_out, stream))


def hyb_attn_step_host(ctx: int, q_host: int, k_host, v_host, out_host: int, stream: int) -> None:
    _check("hyb_attn_step_host", load_library().hyb_attn_step_host(ctx, q_host, k_host, v_host, out_host, stream))


def _ctx_array(ctxs):
    return (c_vp * len(ctxs))(*ctxs)


def hyb_attn_step_layers_staging_bytes(ctxs) -> int:
    return int(load_library().hyb_attn_step_layers_staging_bytes(_ctx_array(ctxs), len(ctxs)))


def hyb_attn_step_layers_host(ctxs, in_host: int, out_host: int, staging: int, staging_bytes: int,
                              stream: int) -> None:
    _check("hyb_attn_step_layers_host",
           load_library().hyb_attn_step_layers_host(_ctx_array(ctxs), len(ctxs), in_host, out_host, staging,
                                                    staging_bytes, stream))


def hyb_attn_decode_noalloc(ctx: int, q: int, out: int, sel_out, stream: int) -> None:
    """Decode with the block scores and the selection in the library's fixed
    device array instead of the context's workspace (for callers that cannot
    allocate device memory)."""
    _check("hyb_attn_decode_noalloc", load_library().hyb_attn_decode_noalloc(ctx, q, out, sel_out, stream))


def hyb_attn_length(ctx: int) -> int:
    return int(load_library().hyb_attn_length(ctx))


def hyb_attn_row_length(ctx: int, b: int) -> int:
    return int(load_library().hyb_attn_row_length(ctx, b))


def hyb_attn_status(ctx: int, clear: bool, stream: int) -> int:
    flags = ctypes.c_uint32(0)
    _check("hyb_attn_status", load_library().hyb_attn_status(ctx, ctypes.byref(flags), int(clear), stream))
    return flags.value


def hyb_attn_set_timing_events(ctx: int, begin, end) -> None:
    _check("hyb_attn_set_timing_events", load_library().hyb_attn_set_timing_events(ctx, begin, end))


def hyb_attn_set_wait_limit(ctx: int, ns: int) -> None:
    _check("hyb_attn_set_wait_limit", load_library().hyb_attn_set_wait_limit(ctx, ns))


def hyb_attn_set_test_flags(ctx: int, flags: int) -> None:
    _check("hyb_attn_set_test_flags", load_library().hyb_attn_set_test_flags(ctx, flags))


def hyb_attn_destroy(ctx: int) -> None:
    load_library().hyb_attn_destroy(ctx)
