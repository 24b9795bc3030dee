"""One attention layer's device buffers (PyTorch-owned) bound to a C-ABI context.

PyTorch is used for device memory and streams only; every step of decode,
append and init runs in the library's kernels.
"""

from __future__ import annotations

import torch

from . import _abi as A


def make_config(batch: int, n_q_heads: int, n_kv_heads: int, head_dim: int, block_size: int, n_sink: int,
                window: int, top_k: int, capacity: int, scale: float = 0.0, head_window=None,
                head_top_k=None) -> A.hyb_attn_config:
    """The C config struct.  With per-KV-head budgets (head_window, head_top_k:
    sequences of n_kv_heads ints), `window` and `top_k` default to their
    minimum and maximum (the sizes the buffers need)."""
    hw = ht = None
    if head_window is not None or head_top_k is not None:
        assert head_window is not None and head_top_k is not None
        assert len(head_window) == n_kv_heads and len(head_top_k) == n_kv_heads
        window = min(window, min(head_window)) if window is not None else min(head_window)
        top_k = max(top_k, max(head_top_k)) if top_k is not None else max(head_top_k)
        hw = (A.c_i32 * n_kv_heads)(*[int(v) for v in head_window])
        ht = (A.c_i32 * n_kv_heads)(*[int(v) for v in head_top_k])
    cfg = A.hyb_attn_config(batch, n_q_heads, n_kv_heads, head_dim, block_size, n_sink, window, top_k,
                            capacity, scale, hw, ht)
    cfg._keep = (hw, ht)   # the arrays live as long as the struct that points at them
    return cfg


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


class HybridAttentionLayer:
    """Caller-owned buffers of one layer plus its library context.

    Buffers (``[B][Hkv]`` leading dims, u = b * Hkv + h):
      k_cache, v_cache bf16 [B, Hkv, capacity, d]; H fp32 [B, Hkv, d, d];
      zk, zv fp32 [B, Hkv, d]; n fp32 [B, Hkv]; mu, var fp32 [B, Hkv, max_blocks, d];
      workspace uint8 (may be shared by layers used on one stream).
    Fill ``k_cache[:, :, :T0]`` / ``v_cache`` with the prefilled history, then call
    ``init(T0)``.
    """

    def __init__(self, cfg: A.hyb_attn_config, device=None, workspace: torch.Tensor | None = None):
        if not torch.cuda.is_available():
            raise RuntimeError("HybridAttentionLayer needs a CUDA device (sm_100a); there is no CPU path")
        self.device = torch.device(device if device is not None else "cuda")
        self.cfg = cfg
        self.sizes = A.hyb_attn_query_sizes(cfg)
        B, Hkv, d, cap = cfg.batch, cfg.n_kv_heads, cfg.head_dim, cfg.capacity
        mb = max(1, self.sizes.max_blocks)
        dev = self.device
        self.k_cache = torch.empty((B, Hkv, cap, d), dtype=torch.bfloat16, device=dev)
        self.v_cache = torch.empty((B, Hkv, cap, d), dtype=torch.bfloat16, device=dev)
        self.H = torch.zeros((B, Hkv, d, d), dtype=torch.float32, device=dev)
        self.zk = torch.zeros((B, Hkv, d), dtype=torch.float32, device=dev)
        self.zv = torch.zeros((B, Hkv, d), dtype=torch.float32, device=dev)
        self.n = torch.zeros((B, Hkv), dtype=torch.float32, device=dev)
        self.mu = torch.zeros((B, Hkv, mb, d), dtype=torch.float32, device=dev)
        self.var = torch.zeros((B, Hkv, mb, d), dtype=torch.float32, device=dev)
        wb = int(self.sizes.workspace_bytes)
        if workspace is None:
            workspace = torch.empty(wb, dtype=torch.uint8, device=dev)
        assert workspace.numel() >= wb
        self.workspace = workspace
        self.ctx = None

    @staticmethod
    def workspace_bytes(cfg: A.hyb_attn_config) -> int:
        return A.hyb_attn_workspace_size(cfg)

    def buffers(self) -> A.hyb_attn_buffers:
        return A.hyb_attn_buffers(self.k_cache.data_ptr(), self.v_cache.data_ptr(), self.H.data_ptr(),
                                  self.zk.data_ptr(), self.zv.data_ptr(), self.n.data_ptr(), self.mu.data_ptr(),
                                  self.var.data_ptr(), self.workspace.data_ptr(), self.workspace.numel())

    def init(self, T0, stream=None) -> None:
        """Build the state of the prefilled history: T0 tokens per row, or a
        sequence of per-row lengths."""
        if self.ctx is not None:
            A.hyb_attn_destroy(self.ctx)
        with torch.cuda.device(self.device):
            if isinstance(T0, int):
                self.ctx = A.hyb_attn_init(self.cfg, self.buffers(), T0, _stream(stream))
            else:
                self.ctx = A.hyb_attn_init_rows(self.cfg, self.buffers(), list(T0), _stream(stream))

    def attach(self, T, stream=None) -> None:
        """Bind a context to buffers that already hold the synced state of a
        history of length T (or per-row lengths): a restored checkpoint,
        without rebuilding it."""
        if self.ctx is not None:
            A.hyb_attn_destroy(self.ctx)
        with torch.cuda.device(self.device):
            if isinstance(T, int):
                self.ctx = A.hyb_attn_attach(self.cfg, self.buffers(), T, _stream(stream))
            else:
                self.ctx = A.hyb_attn_attach_rows(self.cfg, self.buffers(), list(T), _stream(stream))

    def row_lengths(self) -> list:
        return [A.hyb_attn_row_length(self.ctx, b) for b in range(self.cfg.batch)]

    def set_wait_limit(self, ns: int) -> None:
        A.hyb_attn_set_wait_limit(self.ctx, ns)

    def set_test_flags(self, flags: int) -> None:
        A.hyb_attn_set_test_flags(self.ctx, flags)

    @property
    def T(self) -> int:
        return A.hyb_attn_length(self.ctx)

    def decode(self, q: torch.Tensor, out: torch.Tensor | None = None, sel_out: torch.Tensor | None = None,
               scores_out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        c = self.cfg
        assert q.dtype == torch.bfloat16 and q.is_contiguous() and q.shape == (c.batch, c.n_q_heads, c.head_dim)
        if out is None:
            out = torch.empty((c.batch, c.n_q_heads, c.head_dim), dtype=torch.float32, device=q.device)
        if sel_out is not None:
            assert sel_out.dtype == torch.int32 and sel_out.shape == (c.batch, c.n_kv_heads, c.top_k)
        if scores_out is not None:
            assert scores_out.dtype == torch.float32 and scores_out.shape[-1] == max(1, self.sizes.max_blocks)
        A.hyb_attn_decode(self.ctx, q.data_ptr(), out.data_ptr(), _ptr(sel_out), _ptr(scores_out), _stream(stream))
        return out

    def decode_append(self, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                      out: torch.Tensor | None = None, sel_out: torch.Tensor | None = None,
                      scores_out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """Decode at the current T, then append (k_new, v_new): one generation step."""
        c = self.cfg
        assert q.dtype == torch.bfloat16 and q.is_contiguous() and q.shape == (c.batch, c.n_q_heads, c.head_dim)
        for t in (k_new, v_new):
            assert t.dtype == torch.bfloat16 and t.is_contiguous() and t.shape == (c.batch, c.n_kv_heads, c.head_dim)
        if out is None:
            out = torch.empty((c.batch, c.n_q_heads, c.head_dim), dtype=torch.float32, device=q.device)
        if sel_out is not None:
            assert sel_out.dtype == torch.int32 and sel_out.shape == (c.batch, c.n_kv_heads, c.top_k)
        if scores_out is not None:
            assert scores_out.dtype == torch.float32 and scores_out.shape[-1] == max(1, self.sizes.max_blocks)
        A.hyb_attn_decode_append(self.ctx, q.data_ptr(), k_new.data_ptr(), v_new.data_ptr(), out.data_ptr(),
                                 _ptr(sel_out), _ptr(scores_out), _stream(stream))
        return out

    def decode_with_selection(self, q: torch.Tensor, sel: torch.Tensor, out: torch.Tensor | None = None,
                              stream=None) -> torch.Tensor:
        c = self.cfg
        assert sel.dtype == torch.int32 and sel.is_contiguous() and sel.shape == (c.batch, c.n_kv_heads, c.top_k)
        if out is None:
            out = torch.empty((c.batch, c.n_q_heads, c.head_dim), dtype=torch.float32, device=q.device)
        A.hyb_attn_decode_with_selection(self.ctx, q.data_ptr(), sel.data_ptr(), out.data_ptr(), _stream(stream))
        return out

    def decode_strided(self, q: torch.Tensor, k_top: int, stride: int, out: torch.Tensor | None = None,
                       sel_out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """Decode with strided block selection: the last block of every `stride`
        candidate blocks always exact, plus the top-k_top of the others."""
        c = self.cfg
        assert q.dtype == torch.bfloat16 and q.is_contiguous() and q.shape == (c.batch, c.n_q_heads, c.head_dim)
        if out is None:
            out = torch.empty((c.batch, c.n_q_heads, c.head_dim), dtype=torch.float32, device=q.device)
        if sel_out is not None:
            assert sel_out.dtype == torch.int32 and sel_out.shape == (c.batch, c.n_kv_heads, c.top_k)
        A.hyb_attn_decode_strided(self.ctx, q.data_ptr(), int(k_top), int(stride), out.data_ptr(), _ptr(sel_out),
                                  _stream(stream))
        return out

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor, stream=None) -> None:
        c = self.cfg
        for t in (k_new, v_new):
            assert t.dtype == torch.bfloat16 and t.is_contiguous() and t.shape == (c.batch, c.n_kv_heads, c.head_dim)
        A.hyb_attn_append(self.ctx, k_new.data_ptr(), v_new.data_ptr(), _stream(stream))

    def append_chunk(self, k_new: torch.Tensor, v_new: torch.Tensor, stream=None) -> None:
        """Append n tokens per unit in one launch: k_new, v_new [B][Hkv][n][d]."""
        c = self.cfg
        n = k_new.shape[2]
        for t in (k_new, v_new):
            assert t.dtype == torch.bfloat16 and t.is_contiguous() and t.shape == (c.batch, c.n_kv_heads, n, c.head_dim)
        A.hyb_attn_append_chunk(self.ctx, k_new.data_ptr(), v_new.data_ptr(), n, _stream(stream))

    def decode_chunk(self, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                     out: torch.Tensor | None = None, sel_out: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
        """n consecutive decode + append steps: q [n][B][Hq][d], k_new, v_new
        [n][B][Hkv][d]; row j attends to the history and the chunk's tokens
        before j.  Returns out [n][B][Hq][d]."""
        c = self.cfg
        n = q.shape[0]
        assert q.dtype == torch.bfloat16 and q.is_contiguous() and q.shape == (n, c.batch, c.n_q_heads, c.head_dim)
        for t in (k_new, v_new):
            assert t.dtype == torch.bfloat16 and t.is_contiguous() and t.shape == (n, c.batch, c.n_kv_heads, c.head_dim)
        if out is None:
            out = torch.empty((n, c.batch, c.n_q_heads, c.head_dim), dtype=torch.float32, device=q.device)
        if sel_out is not None:
            assert sel_out.dtype == torch.int32 and sel_out.shape == (n, c.batch, c.n_kv_heads, c.top_k)
        A.hyb_attn_decode_chunk(self.ctx, q.data_ptr(), k_new.data_ptr(), v_new.data_ptr(), n, out.data_ptr(),
                                _ptr(sel_out), _stream(stream))
        return out

    def sync_state(self, stream=None) -> None:
        """Fold the evictions since the last decode into H, zk, zv, n, mu, var."""
        A.hyb_attn_sync_state(self.ctx, _stream(stream))

    def step_host(self, q_host: torch.Tensor, k_host, v_host, out_host: torch.Tensor, stream=None) -> None:
        A.hyb_attn_step_host(self.ctx, q_host.data_ptr(), _ptr(k_host), _ptr(v_host), out_host.data_ptr(),
                             _stream(stream))

    def status(self, clear: bool = False, stream=None) -> int:
        return A.hyb_attn_status(self.ctx, clear, _stream(stream))

    def set_timing_events(self, begin: torch.cuda.Event | None, end: torch.cuda.Event | None) -> None:
        A.hyb_attn_set_timing_events(self.ctx, None if begin is None else begin.cuda_event,
                                     None if end is None else end.cuda_event)

    def close(self) -> None:
        if self.ctx is not None:
            A.hyb_attn_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
