"""CPU oracle (fp64) for paged-KV-cache decode attention: Python wrapper.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg may use this package; the product path never does.  It shares
no code with the CUDA path and does not import it.

The arithmetic lives in ``oracle.c`` (plain C, fp64 loops).  This module builds
it with gcc on first use (``build()``), then exposes each C function over
numpy arrays, plus ``caches_for`` / ``decode_for`` helpers that run the oracle
over a workload object (any object with the attributes of
``workload.Workload``).
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

DTYPES = {"f16": 0, "bf16": 1, "e4m3": 2, "e5m2": 3, "int8": 4}
EIGHT_BIT = ("e4m3", "e5m2", "int8")

_lib: Optional[ctypes.CDLL] = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (IEEE arithmetic: no fast-math, no
    contraction, so float division is the correctly rounded one)."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
            "-fexcess-precision=standard", "-o", tmp, _SRC, "-lm",
        ])
        os.replace(tmp, _LIB)
    return _LIB


def use_library(path: Optional[str]) -> None:
    """Load the oracle's functions from another build of oracle.c (the
    mutation tests build copies with a planted mistake); None restores the
    default library."""
    global _lib, _lib_path
    _lib, _lib_path = None, path


_lib_path: Optional[str] = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if _lib_path is None:
            build()
        L = ctypes.CDLL(_lib_path or _LIB)
        P = ctypes.c_void_p
        i32, i64, f32, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_double
        L.orc_f16_decode.restype = f64
        L.orc_f16_decode.argtypes = [ctypes.c_uint16]
        L.orc_bf16_decode.restype = f64
        L.orc_bf16_decode.argtypes = [ctypes.c_uint16]
        L.orc_e4m3_decode.restype = f64
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e4m3_encode.argtypes = [f32]
        L.orc_e5m2_decode.restype = f64
        L.orc_e5m2_decode.argtypes = [ctypes.c_uint8]
        L.orc_e5m2_encode.restype = ctypes.c_uint8
        L.orc_e5m2_encode.argtypes = [f32]
        L.orc_int8_decode.restype = f64
        L.orc_int8_decode.argtypes = [ctypes.c_uint8]
        L.orc_int8_encode.restype = ctypes.c_uint8
        L.orc_int8_encode.argtypes = [f32]
        L.orc_blocks_for_len.restype = i64
        L.orc_blocks_for_len.argtypes = [i64, i32]
        L.orc_kv_bytes_per_token.restype = i64
        L.orc_kv_bytes_per_token.argtypes = [i32, i32, i32, i32]
        L.orc_slot.restype = i64
        L.orc_slot.argtypes = [P, i64, i32]
        L.orc_slot_mapping.restype = None
        L.orc_slot_mapping.argtypes = [P, P, i32, P, P, P, i32, i32]
        L.orc_cache_write.restype = i32
        L.orc_cache_write.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32, f32, f32]
        L.orc_gather.restype = None
        L.orc_gather.argtypes = [P, P, i32, f64, P, i32, i32, i32, i32, i32]
        L.orc_attention.restype = None
        L.orc_attention.argtypes = [P, P, P, P, P, i32, i32, f64]
        L.orc_decode.restype = i32
        L.orc_decode.argtypes = [P, P, i32, P, P, i32, f64, f64, P, i32, P, i32, i32, i32, i32,
                                 i32, f64, P, i32]
        L.orc_split_partials.restype = i32
        L.orc_split_partials.argtypes = [P, P, P, i32, P, P, i32, f64, f64, P, i32, P, i32, i32,
                                         i32, i32, f64, i32, i32, P, i32]
        L.orc_split_merge.restype = None
        L.orc_split_merge.argtypes = [P, P, P, i32, i32]
        L.orc_prefill.restype = i32
        L.orc_prefill.argtypes = [P, P, i32, P, P, i32, f64, f64, P, i32, P, P, i32, i32, i32, i32,
                                  i32, f64]
        L.orc_cache_write_channel.restype = i32
        L.orc_cache_write_channel.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, i32, i32, P, P]
        L.orc_decode_channel.restype = i32
        L.orc_decode_channel.argtypes = [P, P, i32, P, P, i32, P, P, P, i32, P, i32, i32, i32, i32,
                                         i32, f64, P, i32]
        L.orc_copy_blocks.restype = i32
        L.orc_copy_blocks.argtypes = [P, P, P, i32, i32, i32, i32, i32, i32]
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------------------
# element formats
# ---------------------------------------------------------------------------

def f16_decode(bits: int) -> float:
    return lib().orc_f16_decode(int(bits))


def bf16_decode(bits: int) -> float:
    return lib().orc_bf16_decode(int(bits))


def e4m3_decode(code: int) -> float:
    return lib().orc_e4m3_decode(int(code))


def e4m3_encode(y: float) -> int:
    return int(lib().orc_e4m3_encode(float(np.float32(y))))


def e5m2_decode(code: int) -> float:
    return lib().orc_e5m2_decode(int(code))


def e5m2_encode(y: float) -> int:
    return int(lib().orc_e5m2_encode(float(np.float32(y))))


def int8_decode(code: int) -> float:
    return lib().orc_int8_decode(int(code))


def int8_encode(y: float) -> int:
    return int(lib().orc_int8_encode(float(np.float32(y))))


def decode_bits(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Element values of an array of f16 / bf16 / E4M3 / E5M2 / INT8 codes as fp64."""
    fn = {"f16": f16_decode, "bf16": bf16_decode, "e4m3": e4m3_decode, "e5m2": e5m2_decode,
          "int8": int8_decode}[dtype]
    flat = np.asarray(bits).reshape(-1)
    # small arrays only (tests): one C call per element
    return np.array([fn(int(x)) for x in flat], dtype=np.float64).reshape(np.shape(bits))


# ---------------------------------------------------------------------------
# block tables, slots, cache write
# ---------------------------------------------------------------------------

def blocks_for_len(length: int, block_size: int = 16) -> int:
    return int(lib().orc_blocks_for_len(int(length), int(block_size)))


def kv_bytes_per_token(layers: int, kv_heads: int, head_dim: int, bytes_per_elem: int) -> int:
    return int(lib().orc_kv_bytes_per_token(layers, kv_heads, head_dim, bytes_per_elem))


def slot(block_table_row: Sequence[int], pos: int, block_size: int = 16) -> int:
    row = _c(block_table_row, np.int32)
    return int(lib().orc_slot(_p(row), int(pos), int(block_size)))


def slot_mapping(block_tables: np.ndarray, seq_lens: Optional[np.ndarray],
                 token_seq: Optional[np.ndarray], token_pos: Optional[np.ndarray],
                 num_tokens: int, block_size: int = 16) -> np.ndarray:
    bt = _c(block_tables, np.int32)
    sl = None if seq_lens is None else _c(seq_lens, np.int32)
    ts = None if token_seq is None else _c(token_seq, np.int32)
    tp = None if token_pos is None else _c(token_pos, np.int32)
    out = np.empty(num_tokens, dtype=np.int64)
    lib().orc_slot_mapping(_p(out), _p(bt), bt.shape[1], _p(sl), _p(ts), _p(tp), num_tokens,
                           block_size)
    return out


def cache_write(k_new: np.ndarray, v_new: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                slots: np.ndarray, num_blocks: int, num_kv_heads: int, head_dim: int,
                block_size: int, act_dtype: str, kv_dtype: str, k_scale: float = 1.0,
                v_scale: float = 1.0) -> int:
    """In-place write into the numpy pools; returns the number of skipped
    out-of-range slots (raises on an unsupported dtype pair)."""
    kn, vn = _c(k_new, np.uint16), _c(v_new, np.uint16)
    sl = _c(slots, np.int64)
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    r = lib().orc_cache_write(_p(kn), _p(vn), _p(k_cache), _p(v_cache), _p(sl), int(sl.size),
                              num_blocks, num_kv_heads, head_dim, block_size, DTYPES[act_dtype],
                              DTYPES[kv_dtype], float(np.float32(k_scale)),
                              float(np.float32(v_scale)))
    if r < 0:
        raise ValueError("unsupported dtype pair")
    return int(r)


def copy_blocks(k_cache: np.ndarray, v_cache: np.ndarray, pairs: np.ndarray) -> int:
    """In-place copy-on-write block copy inside the numpy pools
    [num_blocks, Hk, B, d]: block dst := block src for every (src, dst) row of
    ``pairs``, in order.  Returns the number of pairs skipped for an
    out-of-range id."""
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    assert k_cache.shape == v_cache.shape and k_cache.dtype == v_cache.dtype
    nb, hk, bs, d = k_cache.shape
    pr = _c(pairs, np.int32).reshape(-1, 2)
    return int(lib().orc_copy_blocks(_p(k_cache), _p(v_cache), _p(pr), pr.shape[0], nb, hk, d,
                                     bs, k_cache.dtype.itemsize))


def cache_write_channel(k_new: np.ndarray, v_new: np.ndarray, k_cache: np.ndarray,
                        v_cache: np.ndarray, slots: np.ndarray, num_blocks: int, num_kv_heads: int,
                        head_dim: int, block_size: int, act_dtype: str, kv_dtype: str,
                        k_scales: np.ndarray, v_scales: np.ndarray) -> int:
    """Cache write into an 8-bit pool with per-channel scales [Hk, d] (fp32)."""
    kn, vn = _c(k_new, np.uint16), _c(v_new, np.uint16)
    sl = _c(slots, np.int64)
    ks, vs = _c(k_scales, np.float32), _c(v_scales, np.float32)
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    r = lib().orc_cache_write_channel(_p(kn), _p(vn), _p(k_cache), _p(v_cache), _p(sl),
                                      int(sl.size), num_blocks, num_kv_heads, head_dim,
                                      block_size, DTYPES[act_dtype], DTYPES[kv_dtype], _p(ks),
                                      _p(vs))
    if r < 0:
        raise ValueError("unsupported dtype pair")
    return int(r)


def empty_pool(num_blocks: int, num_kv_heads: int, block_size: int, head_dim: int, kv_dtype: str,
               fill: int = 0xFF) -> np.ndarray:
    dt = np.uint8 if kv_dtype in EIGHT_BIT else np.uint16
    a = np.empty((num_blocks, num_kv_heads, block_size, head_dim), dtype=dt)
    a.view(np.uint8)[...] = fill
    return a


# ---------------------------------------------------------------------------
# gather + attention
# ---------------------------------------------------------------------------

def gather(cache: np.ndarray, kv_dtype: str, scale: float, block_table_row: np.ndarray,
           length: int, num_kv_heads: int, kvh: int, head_dim: int,
           block_size: int = 16) -> np.ndarray:
    rows = np.empty((max(length, 1), head_dim), dtype=np.float64)
    bt = _c(block_table_row, np.int32)
    lib().orc_gather(_p(rows), _p(cache), DTYPES[kv_dtype], float(scale), _p(bt), int(length),
                     num_kv_heads, kvh, head_dim, block_size)
    return rows[:length]


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray,
              softmax_scale: float) -> Tuple[np.ndarray, float]:
    """Textbook attention of one query row over contiguous fp64 K, V [L, d];
    returns (o, lse)."""
    q, K, V = _c(q, np.float64), _c(K, np.float64), _c(V, np.float64)
    d = q.size
    L = K.shape[0] if K.ndim == 2 else 0
    out = np.empty(d, dtype=np.float64)
    lse = np.zeros(1, dtype=np.float64)
    Kp = K if L else np.zeros((1, d))
    Vp = V if L else np.zeros((1, d))
    lib().orc_attention(_p(out), _p(lse), _p(q), _p(Kp), _p(Vp), L, d, float(softmax_scale))
    return out, float(lse[0])


def decode(q: np.ndarray, q_dtype: str, k_cache: np.ndarray, v_cache: np.ndarray, kv_dtype: str,
           block_tables: np.ndarray, seq_lens: np.ndarray, num_kv_heads: int,
           softmax_scale: float, k_scale: float = 1.0, v_scale: float = 1.0,
           block_size: int = 16, pairs: Optional[np.ndarray] = None) -> np.ndarray:
    """Paged decode attention in fp64.  ``q`` holds [S, Hq, d] 16-bit codes.
    Returns [S, Hq, d], or [len(pairs), d] for the listed (s, h) pairs."""
    q = _c(q, np.uint16)
    S, Hq, d = q.shape
    bt = _c(block_tables, np.int32)
    sl = _c(seq_lens, np.int32)
    pr = None if pairs is None else _c(pairs, np.int32).reshape(-1, 2)
    n = S * Hq if pr is None else pr.shape[0]
    out = np.empty((n, d), dtype=np.float64)
    r = lib().orc_decode(_p(out), _p(q), DTYPES[q_dtype], _p(k_cache), _p(v_cache),
                         DTYPES[kv_dtype], float(k_scale), float(v_scale), _p(bt), bt.shape[1],
                         _p(sl), S, Hq, num_kv_heads, d, block_size, float(softmax_scale),
                         _p(pr), 0 if pr is None else pr.shape[0])
    if r:
        raise ValueError("invalid head configuration")
    return out.reshape(S, Hq, d) if pr is None else out


def decode_channel(q: np.ndarray, q_dtype: str, k_cache: np.ndarray, v_cache: np.ndarray,
                   kv_dtype: str, k_scales: np.ndarray, v_scales: np.ndarray,
                   block_tables: np.ndarray, seq_lens: np.ndarray, num_kv_heads: int,
                   softmax_scale: float, block_size: int = 16,
                   pairs: Optional[np.ndarray] = None) -> np.ndarray:
    """Paged decode attention over an 8-bit cache with per-channel scales."""
    q = _c(q, np.uint16)
    S, Hq, d = q.shape
    bt = _c(block_tables, np.int32)
    sl = _c(seq_lens, np.int32)
    ks, vs = _c(k_scales, np.float32), _c(v_scales, np.float32)
    pr = None if pairs is None else _c(pairs, np.int32).reshape(-1, 2)
    n = S * Hq if pr is None else pr.shape[0]
    out = np.empty((n, d), dtype=np.float64)
    r = lib().orc_decode_channel(_p(out), _p(q), DTYPES[q_dtype], _p(k_cache), _p(v_cache),
                                 DTYPES[kv_dtype], _p(ks), _p(vs), _p(bt), bt.shape[1], _p(sl), S,
                                 Hq, num_kv_heads, d, block_size, float(softmax_scale), _p(pr),
                                 0 if pr is None else pr.shape[0])
    if r:
        raise ValueError("invalid configuration")
    return out.reshape(S, Hq, d) if pr is None else out


def split_partials(q: np.ndarray, q_dtype: str, k_cache: np.ndarray, v_cache: np.ndarray,
                   kv_dtype: str, block_tables: np.ndarray, seq_lens: np.ndarray,
                   num_kv_heads: int, softmax_scale: float, partition_size: int,
                   num_partitions: int, pairs: np.ndarray, k_scale: float = 1.0,
                   v_scale: float = 1.0, block_size: int = 16) -> Tuple[np.ndarray, np.ndarray]:
    """Per-partition (lse [n, NP], o [n, NP, d]) for the listed (s, h) pairs."""
    q = _c(q, np.uint16)
    S, Hq, d = q.shape
    bt = _c(block_tables, np.int32)
    sl = _c(seq_lens, np.int32)
    pr = _c(pairs, np.int32).reshape(-1, 2)
    n = pr.shape[0]
    lse = np.empty((n, num_partitions), dtype=np.float64)
    o = np.empty((n, num_partitions, d), dtype=np.float64)
    r = lib().orc_split_partials(_p(lse), _p(o), _p(q), DTYPES[q_dtype], _p(k_cache),
                                 _p(v_cache), DTYPES[kv_dtype], float(k_scale), float(v_scale),
                                 _p(bt), bt.shape[1], _p(sl), Hq, num_kv_heads, d, block_size,
                                 float(softmax_scale), partition_size, num_partitions, _p(pr), n)
    if r:
        raise ValueError("invalid split configuration")
    return lse, o


def prefill(q: np.ndarray, q_dtype: str, k_cache: np.ndarray, v_cache: np.ndarray,
            kv_dtype: str, block_tables: np.ndarray, seq_lens: np.ndarray,
            query_start: np.ndarray, num_kv_heads: int, softmax_scale: float,
            k_scale: float = 1.0, v_scale: float = 1.0, block_size: int = 16) -> np.ndarray:
    """Chunked-prefill attention in fp64: ``q`` holds [T, Hq, d] 16-bit codes,
    sequence s's chunk is rows query_start[s] .. query_start[s+1] - 1, the
    last tokens of its seq_lens[s]; causal.  Returns [T, Hq, d] (rows no
    sequence covers are 0)."""
    q = _c(q, np.uint16)
    T, Hq, d = q.shape
    bt = _c(block_tables, np.int32)
    sl = _c(seq_lens, np.int32)
    qs = _c(query_start, np.int32)
    out = np.zeros((T, Hq, d), dtype=np.float64)
    r = lib().orc_prefill(_p(out), _p(q), DTYPES[q_dtype], _p(k_cache), _p(v_cache),
                          DTYPES[kv_dtype], float(k_scale), float(v_scale), _p(bt), bt.shape[1],
                          _p(sl), _p(qs), int(sl.size), Hq, num_kv_heads, d, block_size,
                          float(softmax_scale))
    if r:
        raise ValueError("invalid prefill configuration")
    return out


def split_merge(lse: np.ndarray, o: np.ndarray) -> np.ndarray:
    lse, o = _c(lse, np.float64), _c(o, np.float64)
    NP, d = o.shape
    out = np.empty(d, dtype=np.float64)
    lib().orc_split_merge(_p(out), _p(lse), _p(o), NP, d)
    return out


# ---------------------------------------------------------------------------
# whole-workload helpers
# ---------------------------------------------------------------------------

def _write_rows(w, kr, vr, kc, vc, slots):
    if getattr(w, "k_chan", None) is not None:
        cache_write_channel(kr, vr, kc, vc, slots, w.num_blocks, w.num_kv_heads, w.head_dim,
                            w.block_size, w.act_dtype, w.kv_dtype, w.k_chan, w.v_chan)
    else:
        cache_write(kr, vr, kc, vc, slots, w.num_blocks, w.num_kv_heads, w.head_dim,
                    w.block_size, w.act_dtype, w.kv_dtype, w.k_scale, w.v_scale)


def caches_for(w, include_new: bool = True) -> Tuple[np.ndarray, np.ndarray]:
    """The oracle's K/V pools for workload ``w``: poisoned (0xFF) pools, the
    prefill tokens written at their slots, then (``include_new``) this step's
    new token of every sequence at position seq_len - 1.  A workload with
    per-channel scales (``k_chan`` / ``v_chan``) is quantised with them."""
    kc = empty_pool(w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim, w.kv_dtype)
    vc = empty_pool(w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim, w.kv_dtype)
    Tp = int(w.prefill_seq.size)
    if Tp:
        slots = slot_mapping(w.block_tables, w.seq_lens, w.prefill_seq, w.prefill_pos, Tp,
                             w.block_size)
        _write_rows(w, w.k_prefill, w.v_prefill, kc, vc, slots)
    if include_new and w.num_seqs:
        slots = slot_mapping(w.block_tables, w.seq_lens, w.new_seq, None, w.num_seqs,
                             w.block_size)
        _write_rows(w, w.k_new, w.v_new, kc, vc, slots)
    return kc, vc


def chunked_caches_for(w) -> Tuple[np.ndarray, np.ndarray]:
    """The oracle's pools for a chunked-prefill workload (``workload.build_chunked``):
    poisoned pools, then every context token and every chunk token written
    at its slot."""
    kc = empty_pool(w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim, w.kv_dtype)
    vc = empty_pool(w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim, w.kv_dtype)
    for seq, pos, kr, vr in ((w.ctx_seq, w.ctx_pos, w.k_ctx, w.v_ctx),
                             (w.chunk_seq, w.chunk_pos, w.k_chunk, w.v_chunk)):
        T = int(seq.size)
        if T:
            slots = slot_mapping(w.block_tables, None, seq, pos, T, w.block_size)
            cache_write(kr, vr, kc, vc, slots, w.num_blocks, w.num_kv_heads, w.head_dim,
                        w.block_size, w.act_dtype, w.kv_dtype, w.k_scale, w.v_scale)
    return kc, vc


def prefill_for(w, kc: np.ndarray, vc: np.ndarray) -> np.ndarray:
    return prefill(w.q, w.act_dtype, kc, vc, w.kv_dtype, w.block_tables, w.seq_lens,
                   w.query_start, w.num_kv_heads, w.softmax_scale, w.k_scale, w.v_scale,
                   w.block_size)


def decode_for(w, kc: np.ndarray, vc: np.ndarray, pairs: Optional[np.ndarray] = None) -> np.ndarray:
    if getattr(w, "k_chan", None) is not None:
        return decode_channel(w.q, w.act_dtype, kc, vc, w.kv_dtype, w.k_chan, w.v_chan,
                              w.block_tables, w.seq_lens, w.num_kv_heads, w.softmax_scale,
                              w.block_size, pairs)
    return decode(w.q, w.act_dtype, kc, vc, w.kv_dtype, w.block_tables, w.seq_lens,
                  w.num_kv_heads, w.softmax_scale, w.k_scale, w.v_scale, w.block_size, pairs)
