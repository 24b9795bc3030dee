"""numpy implementation of the seeded counter-based generator.

Every draw is a pure function of (seed, stream, element index):

1. ``bits = mix(key(seed, stream) + (index + 1) * GAMMA)`` with the SplitMix64
   finaliser (Steele, Lea and Flood, "Fast splittable pseudorandom number
   generators", OOPSLA 2014) as ``mix``; all arithmetic wraps modulo 2**64.
2. A standard normal by the Box--Muller transform (Box and Muller, 1958) from
   the two 32-bit halves: ``u1 = (hi + 1) / 2**32`` in (0, 1] and ``lo``.
   ``ln(u1)`` and ``cos(2*pi*lo/2**32)`` are evaluated with a fixed series
   (an atanh series for ln, Taylor series for sin/cos after an exact
   quadrant split), using only correctly rounded fp64 operations, so the CUDA
   twin in ``syngen/csrc/syngen.cu`` produces the same bits.
3. Values are formed in fp64, rounded to fp32 (nearest-even), then to bf16
   (nearest-even), exactly as the device side does.
"""

from __future__ import annotations

import numpy as np

from . import configs as C

_M64 = np.uint64(0xFFFFFFFFFFFFFFFF)
GAMMA = 0x9E3779B97F4A7C15
_GAMMA = np.uint64(GAMMA)
_MUL1 = np.uint64(0xBF58476D1CE4E5B9)
_MUL2 = np.uint64(0x94D049BB133111EB)

# Series coefficients as exact doubles (the device file holds the same hex literals).
_LN_COEF = [float.fromhex(h) for h in (
    "0x1.0000000000000p+0", "0x1.5555555555555p-2", "0x1.999999999999ap-3",
    "0x1.2492492492492p-3", "0x1.c71c71c71c71cp-4", "0x1.745d1745d1746p-4",
    "0x1.3b13b13b13b14p-4", "0x1.1111111111111p-4", "0x1.e1e1e1e1e1e1ep-5",
    "0x1.af286bca1af28p-5", "0x1.8618618618618p-5", "0x1.642c8590b2164p-5")]
_COS_COEF = [float.fromhex(h) for h in (
    "0x1.0000000000000p+0", "-0x1.0000000000000p-1", "0x1.5555555555555p-5",
    "-0x1.6c16c16c16c17p-10", "0x1.a01a01a01a01ap-16", "-0x1.27e4fb7789f5cp-22",
    "0x1.1eed8eff8d898p-29", "-0x1.93974a8c07c9dp-37", "0x1.ae7f3e733b81fp-45",
    "-0x1.6827863b97d97p-53", "0x1.e542ba4020225p-62", "-0x1.0ce396db7f853p-70",
    "0x1.f2cf01972f578p-80")]
_SIN_COEF = [float.fromhex(h) for h in (
    "0x1.0000000000000p+0", "-0x1.5555555555555p-3", "0x1.1111111111111p-7",
    "-0x1.a01a01a01a01ap-13", "0x1.71de3a556c734p-19", "-0x1.ae64567f544e4p-26",
    "0x1.6124613a86d09p-33", "-0x1.ae7f3e733b81fp-41", "0x1.952c77030ad4ap-49",
    "-0x1.2f49b46814157p-57", "0x1.71b8ef6dcf572p-66", "-0x1.761b41316381ap-75",
    "0x1.3f3ccdd165fa9p-84")]
_LN2 = float.fromhex("0x1.62e42fefa39efp-1")
_HALF_PI = float.fromhex("0x1.921fb54442d18p+0")
_SQRT_HALF = float.fromhex("0x1.6a09e667f3bcdp-1")
_TWO_M32 = 2.0 ** -32
_TWO_M30 = 2.0 ** -30
_TWO_M53 = 2.0 ** -53


def _mix_scalar(z: int) -> int:
    m = (1 << 64) - 1
    z &= m
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & m
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & m
    return z ^ (z >> 31)


def stream_key(seed: int, stream: int) -> int:
    """64-bit key of one stream: mixes the seed and the stream id."""
    m = (1 << 64) - 1
    return _mix_scalar((seed * GAMMA + stream * 0xD1B54A32D192ED03 + 0x632BE59BD9B4E019) & m)


def raw_bits(key: int, idx: np.ndarray) -> np.ndarray:
    """SplitMix64 output for element indices ``idx`` (uint64 array)."""
    idx = np.asarray(idx, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + (idx + np.uint64(1)) * _GAMMA
        z = (z ^ (z >> np.uint64(30))) * _MUL1
        z = (z ^ (z >> np.uint64(27))) * _MUL2
    return z ^ (z >> np.uint64(31))


def _ln_unit(hi: np.ndarray) -> np.ndarray:
    """ln((hi + 1) * 2**-32) for 32-bit integers ``hi``."""
    n = hi.astype(np.float64) + 1.0                  # exact: integer in [1, 2**32]
    m, e = np.frexp(n)                               # n = m * 2**e, m in [0.5, 1)
    small = m < _SQRT_HALF
    m = np.where(small, m * 2.0, m)                  # exact
    e = np.where(small, e - 1, e).astype(np.float64)
    t = (m - 1.0) / (m + 1.0)
    t2 = t * t
    p = np.full_like(t, _LN_COEF[-1])
    for c in _LN_COEF[-2::-1]:
        p = p * t2
        p = p + c
    ln_m = (t * 2.0) * p
    return (e - 32.0) * _LN2 + ln_m


def _cos_turn(lo: np.ndarray) -> np.ndarray:
    """cos(2*pi * lo * 2**-32) for 32-bit integers ``lo``."""
    quad = (lo >> np.uint64(30)).astype(np.int64)
    frac = (lo & np.uint64(0x3FFFFFFF)).astype(np.float64) * _TWO_M30
    th = frac * _HALF_PI
    t2 = th * th
    pc = np.full_like(th, _COS_COEF[-1])
    for c in _COS_COEF[-2::-1]:
        pc = pc * t2
        pc = pc + c
    ps = np.full_like(th, _SIN_COEF[-1])
    for c in _SIN_COEF[-2::-1]:
        ps = ps * t2
        ps = ps + c
    ps = ps * th
    out = np.where(quad == 0, pc, np.where(quad == 1, -ps, np.where(quad == 2, -pc, ps)))
    return out


def _normal_chunk(key: int, idx: np.ndarray) -> np.ndarray:
    b = raw_bits(key, idx)
    hi = b >> np.uint64(32)
    lo = b & np.uint64(0xFFFFFFFF)
    r = np.sqrt(_ln_unit(hi) * -2.0)
    return r * _cos_turn(lo)


_CHUNK = 1 << 15


def normal(key: int, idx: np.ndarray) -> np.ndarray:
    """Standard normal draws (fp64) for element indices ``idx`` (any shape)."""
    idx = np.asarray(idx, dtype=np.uint64)
    flat = idx.reshape(-1)
    n = flat.size
    if n <= _CHUNK:
        return _normal_chunk(key, flat).reshape(idx.shape)
    out = np.empty(n, dtype=np.float64)

    def work(s):
        out[s:s + _CHUNK] = _normal_chunk(key, flat[s:s + _CHUNK])

    with _pool() as ex:
        list(ex.map(work, range(0, n, _CHUNK)))
    return out.reshape(idx.shape)


def _pool():
    import concurrent.futures
    import os
    return concurrent.futures.ThreadPoolExecutor(max_workers=max(1, min(32, os.cpu_count() or 1)))


def uniform(key: int, idx: np.ndarray) -> np.ndarray:
    """Uniform draws in [0, 1) with 53 random bits."""
    b = raw_bits(key, idx)
    return (b >> np.uint64(11)).astype(np.float64) * _TWO_M53


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 -> fp32 (nearest-even) -> bf16 (nearest-even); returns uint16 bits."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return u.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------- workload tables

def head_scales(w: C.Workload) -> np.ndarray:
    """[layers][n_kv_heads] fp64 scale, U(0.5, 2) per (layer, kv head), else ones."""
    if not w.head_scale:
        return np.ones((w.layers, w.n_kv_heads), dtype=np.float64)
    idx = np.arange(w.layers * w.n_kv_heads, dtype=np.uint64)
    u = uniform(stream_key(w.seed, C.STREAM_HEAD_SCALE), idx)
    return (0.5 + 1.5 * u).reshape(w.layers, w.n_kv_heads)


def q_bits(w: C.Workload, layer: int, step: int) -> np.ndarray:
    """Query of one decode step: [batch][n_q_heads][head_dim] bf16 bits."""
    n = w.batch * w.n_q_heads * w.head_dim
    base = (layer * C.STEP_STRIDE + step) * n
    idx = np.arange(base, base + n, dtype=np.uint64)
    z = normal(stream_key(w.seed, C.STREAM_Q), idx)
    return f64_to_bf16_bits(z).reshape(w.batch, w.n_q_heads, w.head_dim)


def q_hat(w: C.Workload, layer: int) -> np.ndarray:
    """[batch][n_kv_heads][head_dim] fp64 unit vector of the group-summed step-0 query."""
    q = bf16_bits_to_f64(q_bits(w, layer, 0)).reshape(w.batch, w.n_kv_heads, w.group, w.head_dim)
    s = q.sum(axis=2)
    return s / np.sqrt((s * s).sum(axis=-1, keepdims=True))


def planted_blocks(w: C.Workload, layer: int) -> np.ndarray:
    """[batch][n_kv_heads][n_planted] int32: seeded distinct full-block indices at step 0."""
    nfull = w.evicted(w.T0) // w.block_size
    if w.n_planted == 0:
        return np.zeros((w.batch, w.n_kv_heads, 0), dtype=np.int32)
    assert nfull >= w.n_planted
    key = stream_key(w.seed, C.STREAM_PLANTED)
    out = np.empty((w.batch, w.n_kv_heads, w.n_planted), dtype=np.int32)
    for b in range(w.batch):
        for h in range(w.n_kv_heads):
            unit = (layer * w.batch + b) * w.n_kv_heads + h
            idx = np.uint64(unit) * np.uint64(C.BLOCK_STRIDE) + np.arange(nfull, dtype=np.uint64)
            r = raw_bits(key, idx)
            order = np.lexsort((np.arange(nfull), r))
            out[b, h] = np.sort(order[: w.n_planted])
    return out


class LayerTables:
    """Host-computed per-layer tables both generator twins consume."""

    def __init__(self, w: C.Workload, layer: int):
        self.w = w
        self.layer = layer
        self.scale = head_scales(w)[layer]                       # [Hkv]
        self.planted = planted_blocks(w, layer)                   # [B][Hkv][P]
        self.qhat = q_hat(w, layer) if w.n_planted else np.zeros(
            (w.batch, w.n_kv_heads, w.head_dim))


def kv_bits(w: C.Workload, tables: LayerTables, b: int, h: int, t0: int, t1: int):
    """Keys and values of positions [t0, t1) of (layer, b, kv head): two [n][d] uint16 arrays."""
    d = w.head_dim
    layer = tables.layer
    unit = (layer * w.batch + b) * w.n_kv_heads + h
    n = t1 - t0
    pos = np.arange(t0, t1, dtype=np.int64)
    idx = ((np.uint64(unit) * np.uint64(C.TOKEN_STRIDE) + pos.astype(np.uint64))[:, None]
           * np.uint64(d) + np.arange(d, dtype=np.uint64)[None, :])
    zk = normal(stream_key(w.seed, C.STREAM_K), idx)
    zv = normal(stream_key(w.seed, C.STREAM_V), idx)
    base = zk
    rel = pos - w.n_sink
    blk = np.where(rel >= 0, rel // w.block_size, -1)
    if w.n_planted:
        ev0 = w.n_sink + w.evicted(w.T0)
        planted = np.isin(blk, tables.planted[b, h]) & (pos >= w.n_sink) & (pos < ev0)
        if planted.any():
            pv = tables.qhat[b, h][None, :] * w.planted_amp + zk * w.planted_std
            base = np.where(planted[:, None], pv, base)
    if w.block_offset_std > 0:
        oidx = ((np.uint64(unit) * np.uint64(C.BLOCK_STRIDE)
                 + np.maximum(blk, 0).astype(np.uint64))[:, None] * np.uint64(d)
                + np.arange(d, dtype=np.uint64)[None, :])
        zo = normal(stream_key(w.seed, C.STREAM_BLOCK_OFFSET), oidx)
        base = np.where((blk >= 0)[:, None], base + zo * w.block_offset_std, base)
    s = tables.scale[h]
    kb = f64_to_bf16_bits(base * s)
    vb = f64_to_bf16_bits(zv * s)
    assert kb.shape == (n, d)
    return kb, vb


def kv_f64(w, tables, b, h, t0, t1):
    kb, vb = kv_bits(w, tables, b, h, t0, t1)
    return bf16_bits_to_f64(kb), bf16_bits_to_f64(vb)
