"""The C-ABI library builds, loads and exports every entry point the header
declares; host-only entry points (sizes, plan, argument checks) work without a
GPU.  No kernel is launched here."""

import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hyb_attn.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(hyb_attn_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from hybrid_sparse_linear_decode_b200 import build
    build.build()
    from hybrid_sparse_linear_decode_b200 import _abi
    return _abi.load_library()


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ["hyb_attn_init", "hyb_attn_append", "hyb_attn_decode", "hyb_attn_decode_with_selection",
              "hyb_attn_workspace_size", "hyb_attn_length", "hyb_attn_status", "hyb_attn_destroy",
              "hyb_attn_strerror", "hyb_attn_query_sizes", "hyb_attn_plan", "hyb_attn_step_host",
              "hyb_attn_set_timing_events", "hyb_attn_decode_append", "hyb_attn_sync_state",
              "hyb_attn_attach", "hyb_attn_set_wait_limit", "hyb_attn_set_test_flags",
              "hyb_attn_init_rows", "hyb_attn_attach_rows", "hyb_attn_row_length"]:
        assert n in names, n


def test_documented_departures_from_the_first_boundary_sketch():
    """Two departures from the first sketch of the boundary, documented in the
    header: the status call takes (ctx, uint32_t* flags, int clear, stream),
    and the buffers hold no open-block running sums (the open block's mean /
    variance rows are updated in place)."""
    src = open(HEADER).read()
    flat = re.sub(r"\s+", " ", re.sub(r"/\*.*?\*/", "", src, flags=re.S))
    assert "int hyb_attn_status(hyb_attn_ctx* ctx, uint32_t* flags, int clear, cudaStream_t stream);" in flat
    body = re.search(r"typedef struct hyb_attn_buffers \{(.*?)\} hyb_attn_buffers;", flat).group(1)
    fields = re.findall(r"(\w+);", body)
    assert fields == ["k_cache", "v_cache", "H", "zk", "zv", "n", "mu", "var", "workspace", "workspace_bytes"]
    assert "open_sum" not in flat and "open_sq" not in flat
    assert "Welford" in src and "hyb_attn_status" in src


def test_library_exports_every_declared_symbol(lib):
    from hybrid_sparse_linear_decode_b200 import _abi
    so = _abi.LIB_PATH
    out = subprocess.run(["nm", "-D", "--defined-only", so], capture_output=True, text=True, check=True).stdout
    exported = set(l.split()[-1] for l in out.splitlines() if l.strip())
    for n in _declared_functions():
        assert n in exported, f"{n} declared in hyb_attn.h but not exported"
        assert getattr(lib, n) is not None
    # the binding covers the same set
    assert set(n for n, _, _ in _abi.SIGNATURES) == set(_declared_functions())


def _cfg(**kw):
    from hybrid_sparse_linear_decode_b200 import make_config
    base = dict(batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128, block_size=64, n_sink=4, window=1024,
                top_k=16, capacity=32768 + 64)
    base.update(kw)
    return make_config(**base)


def test_sizes_and_workspace(lib):
    import hybrid_sparse_linear_decode_b200 as H
    c = _cfg()
    s = H.hyb_attn_query_sizes(c)
    assert s.kv_cache_elems == 8 * (32768 + 64) * 128
    assert s.H_elems == 8 * 128 * 128 and s.z_elems == 8 * 128 and s.n_elems == 8
    assert s.max_blocks == -(-(32768 + 64 - 4 - 1024) // 64)
    assert s.stats_elems == 8 * s.max_blocks * 128
    assert s.workspace_bytes == H.hyb_attn_workspace_size(c) > 0
    # window and sinks covering the whole capacity: no blocks at all
    s2 = H.hyb_attn_query_sizes(_cfg(capacity=1000))
    assert s2.max_blocks == 0


@pytest.mark.parametrize("bad", [dict(head_dim=96), dict(n_q_heads=24, n_kv_heads=8), dict(n_q_heads=64),
                                 dict(block_size=0), dict(top_k=-1), dict(capacity=0), dict(window=-1),
                                 dict(scale=-1.0), dict(batch=4096, capacity=1 << 20)])
def test_invalid_configs_rejected(lib, bad):
    import hybrid_sparse_linear_decode_b200 as H
    with pytest.raises(H.HybAttnError) as e:
        H.hyb_attn_query_sizes(_cfg(**bad))
    assert e.value.code == -1
    assert H.hyb_attn_workspace_size(_cfg(**bad)) == 0


def test_init_rejects_bad_arguments_without_touching_a_gpu(lib):
    import hybrid_sparse_linear_decode_b200 as H
    c = _cfg()
    buf = H.hyb_attn_buffers()  # all null
    with pytest.raises(H.HybAttnError) as e:
        H.hyb_attn_init(c, buf, 100, 0)
    assert e.value.code == -1
    buf2 = H.hyb_attn_buffers(16, 32, 48, 64, 80, 96, 112, 128, 256, 1)  # tiny workspace
    with pytest.raises(H.HybAttnError):
        H.hyb_attn_init(c, buf2, 100, 0)
    with pytest.raises(H.HybAttnError):
        H.hyb_attn_init(c, buf2, c.capacity + 1, 0)
    # null context handles
    assert lib.hyb_attn_decode(None, None, None, None, None, None) == -1
    assert lib.hyb_attn_append(None, None, None, None) == -1
    assert lib.hyb_attn_append_chunk(None, None, None, 4, None) == -1
    assert lib.hyb_attn_decode_chunk(None, None, None, None, 4, None, None, None) == -1
    assert lib.hyb_attn_length(None) == -1
    assert lib.hyb_attn_set_wait_limit(None, 0) == -1
    assert lib.hyb_attn_set_test_flags(None, 0) == -1
    with pytest.raises(H.HybAttnError):
        H.hyb_attn_attach(c, buf, 100, 0)
    assert H.hyb_attn_strerror(-2).startswith("KV cache capacity")


@pytest.mark.parametrize("T", [0, 1, 3, 4, 5, 1027, 1028, 1029, 1092, 1093, 32768, 32768 + 64])
def test_plan_partition(lib, T):
    """Chunk counts of the exact set follow the partition (sinks, window, and
    ceil(Bk/64) chunks per selected block); each unit gets one cluster of at
    most 16 CTAs, as many as keep the grid within one CTA per SM."""
    import hybrid_sparse_linear_decode_b200 as H
    c = _cfg()
    n_sm = 148
    p = H.hyb_attn_plan(c, T, n_sm)
    S, W, Bk, units = 4, 1024, 64, 8
    ev = max(0, T - S - W)
    nb = -(-ev // Bk)
    assert p.n_blocks == nb and p.k_eff == min(16, nb)
    sink = min(S, T)
    win = T - max(S, T - W) if T > S else 0
    assert p.chunks_per_unit == -(-sink // 64) + -(-win // 64) + p.k_eff
    assert p.cluster_ctas == 16 and p.grid_ctas == units * 16


@pytest.mark.parametrize("batch,want", [(1, 16), (2, 9), (4, 4), (8, 2), (16, 1), (512, 1)])
def test_plan_cluster_size(lib, batch, want):
    """8 KV heads per row on 148 SMs: min(16, floor(148 / units)) CTAs per unit."""
    import hybrid_sparse_linear_decode_b200 as H
    c = _cfg(batch=batch, capacity=4096)
    p = H.hyb_attn_plan(c, 4096, 148)
    assert p.cluster_ctas == want and p.grid_ctas == batch * 8 * want


def test_per_head_budgets_validated_on_the_host(lib):
    """Per-KV-head budgets refine the config's (window, top_k): every head's
    window at least `window` (which sizes the statistics arrays), every head's
    top-k at most `top_k` (the selection rows' length); at most 32 KV heads."""
    import hybrid_sparse_linear_decode_b200 as H
    ok = H.make_config(1, 32, 8, 128, 64, 4, None, None, 40000, head_window=[1024, 2048] * 4,
                       head_top_k=[16, 32] * 4)
    assert (ok.window, ok.top_k) == (1024, 32)
    s_ok = H.hyb_attn_query_sizes(ok)
    assert s_ok.max_blocks == -(-(40000 - 4 - 1024) // 64)
    bad = H.make_config(1, 32, 8, 128, 64, 4, None, None, 40000, head_window=[1024, 2048] * 4,
                        head_top_k=[16, 32] * 4)
    bad.window = 2000                       # a head below the config's window
    with pytest.raises(H.HybAttnError):
        H.hyb_attn_query_sizes(bad)
    bad2 = H.make_config(1, 32, 8, 128, 64, 4, None, None, 40000, head_window=[1024] * 8, head_top_k=[16] * 8)
    bad2.top_k = 8                          # a head above the config's top-k
    with pytest.raises(H.HybAttnError):
        H.hyb_attn_query_sizes(bad2)
    many = H.make_config(1, 64, 64, 128, 64, 4, None, None, 4096, head_window=[64] * 64, head_top_k=[4] * 64)
    with pytest.raises(H.HybAttnError):    # more KV heads than per-head budgets are kept for
        H.hyb_attn_query_sizes(many)
    half = H.make_config(1, 32, 8, 128, 64, 4, 64, 4, 4096)
    import ctypes
    half.head_window = (ctypes.c_int32 * 8)(*([64] * 8))   # one array without the other
    with pytest.raises(H.HybAttnError):
        H.hyb_attn_query_sizes(half)


def test_per_row_entry_points_reject_bad_arguments(lib):
    import hybrid_sparse_linear_decode_b200 as H
    c = _cfg(batch=2)
    buf = H.hyb_attn_buffers()
    with pytest.raises(H.HybAttnError):
        H.hyb_attn_init_rows(c, buf, [100, 200], 0)          # null buffers
    assert lib.hyb_attn_init_rows(None, None, None, None, None) == -1
    assert lib.hyb_attn_attach_rows(None, None, None, None, None) == -1
    assert lib.hyb_attn_row_length(None, 0) == -1
