"""B200-native paged KV cache decode: Python binding of libpa369.so.

Argument marshalling only: every function here forwards to the C ABI of the
same name (include/pa.h), whose kernels do all of the work.  Tensors are torch
CUDA tensors (device memory and streams come from PyTorch); integer pointers
are accepted too.  A non-OK status raises ``PaError``.

The shared library is built in-tree by ``python paged_kv_cache_369_b200/build.py``;
importing this package without it (or with a stale one) raises ImportError:
there is no fallback.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Union

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa369.so")

PA_OK = 0
PA_ERR_INVALID_ARG = 1
PA_ERR_UNSUPPORTED = 2
PA_ERR_CUDA = 3
PA_ERR_DEVICE_BOUNDS = 4
PA_ERR_DEVICE_TIMEOUT = 5

PA_F16 = 0
PA_BF16 = 1
PA_FP8_E4M3 = 2
PA_FP8_E5M2 = 3
PA_INT8 = 4

# every extern "C" symbol declared in include/pa.h
SYMBOLS = (
    "pa_status_string", "pa_version", "pa_slot_mapping", "pa_cache_write", "pa_decode",
    "pa_split_workspace_bytes", "pa_decode_split_reduce", "pa_decode_split_reduce_static_scratch",
    "pa_decode_append", "pa_copy_blocks", "pa_prefill", "pa_cache_write_per_channel",
    "pa_decode_per_channel", "pa_shared_prefix_workspace_bytes", "pa_decode_shared_prefix",
)

PA_STATIC_SCRATCH_BYTES = 32 * 1024 * 1024


class PaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {pa_status_string(status)}")


if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python paged_kv_cache_369_b200/build.py` "
        "(nvcc, sm_100a). There is no CPU fallback.")

_lib = ctypes.CDLL(LIB_PATH)
_missing = [name for name in SYMBOLS if not hasattr(_lib, name)]
if _missing:
    raise ImportError(f"{LIB_PATH} is stale (missing {', '.join(_missing)}): rebuild it with "
                      "`python paged_kv_cache_369_b200/build.py`")
_P, _I, _F, _S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t

_lib.pa_status_string.restype = ctypes.c_char_p
_lib.pa_status_string.argtypes = [_I]
_lib.pa_version.restype = _I
_lib.pa_version.argtypes = []
_lib.pa_slot_mapping.restype = _I
_lib.pa_slot_mapping.argtypes = [_P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _P, _P]
_lib.pa_cache_write.restype = _I
_lib.pa_cache_write.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _F, _P, _P]
_lib.pa_decode.restype = _I
_lib.pa_decode.argtypes = [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _F,
                           _F, _P, _P]
_lib.pa_split_workspace_bytes.restype = _S
_lib.pa_split_workspace_bytes.argtypes = [_I, _I, _I, _I, _I]
_lib.pa_decode_split_reduce.restype = _I
_lib.pa_decode_split_reduce.argtypes = [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _F,
                                        _I, _I, _F, _F, _I, _I, _P, _S, _P, _P]
_lib.pa_decode_append.restype = _I
_lib.pa_decode_append.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _F,
                                  _I, _I, _F, _F, _I, _I, _P, _S, _P, _P]
_lib.pa_decode_split_reduce_static_scratch.restype = _I
_lib.pa_decode_split_reduce_static_scratch.argtypes = [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I,
                                                       _I, _I, _F, _I, _I, _F, _F, _I, _I, _P, _P]
_lib.pa_prefill.restype = _I
_lib.pa_prefill.argtypes = [_P, _P, _P, _P, _P, _I, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F,
                            _I, _I, _F, _F, _P, _P]
_lib.pa_cache_write_per_channel.restype = _I
_lib.pa_cache_write_per_channel.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P,
                                            _P, _P]
_lib.pa_decode_per_channel.restype = _I
_lib.pa_decode_per_channel.argtypes = [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _F, _I,
                                       _I, _P, _P, _I, _I, _P, _S, _P, _P]
_lib.pa_shared_prefix_workspace_bytes.restype = _S
_lib.pa_shared_prefix_workspace_bytes.argtypes = [_I, _I, _I, _I, _I, _I]
_lib.pa_decode_shared_prefix.restype = _I
_lib.pa_decode_shared_prefix.argtypes = [_P, _P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _F,
                                         _I, _I, _F, _F, _I, _I, _I, _P, _S, _P, _P]
_lib.pa_copy_blocks.restype = _I
_lib.pa_copy_blocks.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P]


def lib() -> ctypes.CDLL:
    """The loaded libpa369.so with its argument types set."""
    return _lib


Ptr = Union[None, int, "torch.Tensor"]  # noqa: F821


def _ptr(x: Ptr) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str) -> None:
    if status != PA_OK:
        raise PaError(status, where)


def dtype_code(dtype) -> int:
    """pa_dtype of a torch dtype: float16, bfloat16, float8_e4m3fn (or uint8
    storage: E4M3 codes), float8_e5m2, int8."""
    import torch

    if dtype == torch.float16:
        return PA_F16
    if dtype == torch.bfloat16:
        return PA_BF16
    if dtype in (torch.uint8, getattr(torch, "float8_e4m3fn", None)):
        return PA_FP8_E4M3
    if dtype == getattr(torch, "float8_e5m2", None):
        return PA_FP8_E5M2
    if dtype == torch.int8:
        return PA_INT8
    raise ValueError(f"no pa_dtype for {dtype}")


def pool_torch_dtype(kv: str):
    """torch storage dtype of each cache format, for pools allocated in Python."""
    import torch

    return {"f16": torch.float16, "bf16": torch.bfloat16, "e4m3": torch.uint8,
            "e5m2": torch.float8_e5m2, "int8": torch.int8}[kv]


def pa_status_string(status: int) -> str:
    return _lib.pa_status_string(int(status)).decode()


def pa_version() -> int:
    return int(_lib.pa_version())


def pa_slot_mapping(slot_mapping, block_tables, seq_lens, token_seq, token_pos, num_tokens: int,
                    num_seqs: int, num_blocks: int, block_size: int = 16, dev_err=None,
                    stream=None) -> None:
    mbs = int(block_tables.shape[1]) if hasattr(block_tables, "shape") else 0
    _check(_lib.pa_slot_mapping(_ptr(slot_mapping), _ptr(block_tables), mbs, _ptr(seq_lens),
                                _ptr(token_seq), _ptr(token_pos), int(num_tokens), int(num_seqs),
                                int(block_size), int(num_blocks), _ptr(dev_err), _stream(stream)),
           "pa_slot_mapping")


def pa_cache_write(k_new, v_new, k_cache, v_cache, slot_mapping, k_scale: float = 1.0,
                   v_scale: float = 1.0, dev_err=None, stream=None) -> None:
    T, Hk, d = (int(x) for x in k_new.shape)
    nb, _, B, _ = (int(x) for x in k_cache.shape)
    _check(_lib.pa_cache_write(_ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                               _ptr(slot_mapping), T, nb, Hk, d, B, dtype_code(k_new.dtype),
                               dtype_code(k_cache.dtype), float(k_scale), float(v_scale),
                               _ptr(dev_err), _stream(stream)),
           "pa_cache_write")


def pa_decode(out, q, k_cache, v_cache, block_tables, seq_lens, softmax_scale: float,
              k_scale: float = 1.0, v_scale: float = 1.0, dev_err=None, stream=None) -> None:
    S, Hq, d = (int(x) for x in q.shape)
    nb, Hk, B, _ = (int(x) for x in k_cache.shape)
    _check(_lib.pa_decode(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                          int(block_tables.shape[1]), _ptr(seq_lens), S, Hq, Hk, d, B, nb,
                          float(softmax_scale), dtype_code(q.dtype), dtype_code(k_cache.dtype),
                          float(k_scale), float(v_scale), _ptr(dev_err), _stream(stream)),
           "pa_decode")


def pa_split_workspace_bytes(num_seqs: int, num_q_heads: int, head_dim: int, max_seq_len: int,
                             partition_size: int) -> int:
    return int(_lib.pa_split_workspace_bytes(num_seqs, num_q_heads, head_dim, max_seq_len,
                                             partition_size))


def pa_decode_split_reduce(out, q, k_cache, v_cache, block_tables, seq_lens,
                           softmax_scale: float, partition_size: int, max_seq_len: int,
                           workspace, k_scale: float = 1.0, v_scale: float = 1.0, dev_err=None,
                           stream=None) -> None:
    S, Hq, d = (int(x) for x in q.shape)
    nb, Hk, B, _ = (int(x) for x in k_cache.shape)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(_lib.pa_decode_split_reduce(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                       _ptr(block_tables), int(block_tables.shape[1]),
                                       _ptr(seq_lens), S, Hq, Hk, d, B, nb, float(softmax_scale),
                                       dtype_code(q.dtype), dtype_code(k_cache.dtype),
                                       float(k_scale), float(v_scale), int(partition_size),
                                       int(max_seq_len), _ptr(workspace), ws_bytes,
                                       _ptr(dev_err), _stream(stream)),
           "pa_decode_split_reduce")


def pa_decode_append(out, q, k_new, v_new, k_cache, v_cache, block_tables, seq_lens,
                     softmax_scale: float, partition_size: int, max_seq_len: int, workspace=None,
                     k_scale: float = 1.0, v_scale: float = 1.0, dev_err=None,
                     stream=None) -> None:
    """One decode step: store each sequence's new token, then attend
    (partition_size 0: single pass; > 0: split-KV with ``workspace``)."""
    S, Hq, d = (int(x) for x in q.shape)
    nb, Hk, B, _ = (int(x) for x in k_cache.shape)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.pa_decode_append(_ptr(out), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
                                 _ptr(v_cache), _ptr(block_tables), int(block_tables.shape[1]),
                                 _ptr(seq_lens), S, Hq, Hk, d, B, nb, float(softmax_scale),
                                 dtype_code(q.dtype), dtype_code(k_cache.dtype), float(k_scale),
                                 float(v_scale), int(partition_size), int(max_seq_len),
                                 _ptr(workspace), ws_bytes, _ptr(dev_err), _stream(stream)),
           "pa_decode_append")


def split_workspace_views(workspace, num_seqs: int, num_q_heads: int, head_dim: int,
                          max_seq_len: int, partition_size: int):
    """(lse [S, Hq, NP], o [S, Hq, NP, d]) fp32 views of a split workspace, in
    the layout pa.h documents."""
    import torch

    np_ = max(1, -(-max_seq_len // partition_size)) if max_seq_len > 0 else 1
    rows = num_seqs * num_q_heads * np_
    lse_bytes = (rows * 4 + 255) // 256 * 256
    flat = workspace.view(torch.uint8)
    lse = flat[:rows * 4].view(torch.float32).view(num_seqs, num_q_heads, np_)
    o = flat[lse_bytes:lse_bytes + rows * head_dim * 4].view(torch.float32)
    return lse, o.view(num_seqs, num_q_heads, np_, head_dim)


def pa_decode_split_reduce_static_scratch(out, q, k_cache, v_cache, block_tables, seq_lens,
                                          softmax_scale: float, partition_size: int,
                                          max_seq_len: int, k_scale: float = 1.0,
                                          v_scale: float = 1.0, dev_err=None,
                                          stream=None) -> None:
    """Split-KV decode whose partials live in the library's own device array
    (PA_STATIC_SCRATCH_BYTES), for callers that cannot allocate; see pa.h."""
    S, Hq, d = (int(x) for x in q.shape)
    nb, Hk, B, _ = (int(x) for x in k_cache.shape)
    _check(_lib.pa_decode_split_reduce_static_scratch(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        int(block_tables.shape[1]), _ptr(seq_lens), S, Hq, Hk, d, B, nb, float(softmax_scale),
        dtype_code(q.dtype), dtype_code(k_cache.dtype), float(k_scale), float(v_scale),
        int(partition_size), int(max_seq_len), _ptr(dev_err), _stream(stream)),
        "pa_decode_split_reduce_static_scratch")


def pa_copy_blocks(k_cache, v_cache, block_pairs, dev_err=None, stream=None) -> None:
    """Copy-on-write block copy: block dst := block src in both pools for
    every (src, dst) row of ``block_pairs`` (device int32 [n, 2])."""
    nb, Hk, B, d = (int(x) for x in k_cache.shape)
    n = int(block_pairs.shape[0]) if block_pairs is not None else 0
    _check(_lib.pa_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(block_pairs), n, nb, Hk, d, B,
                               dtype_code(k_cache.dtype), _ptr(dev_err), _stream(stream)),
           "pa_copy_blocks")


def pa_prefill(out, q, k_cache, v_cache, block_tables, seq_lens, query_start, max_query_len: int,
               softmax_scale: float, dev_err=None, stream=None, k_scale: float = 1.0,
               v_scale: float = 1.0) -> None:
    """Chunked-prefill attention: the rows query_start[s] .. query_start[s+1]-1
    of ``q`` ([T, Hq, d]) are the last tokens of sequence s's seq_lens[s] and
    attend causally over its cache."""
    T, Hq, d = (int(x) for x in q.shape)
    nb, Hk, B, _ = (int(x) for x in k_cache.shape)
    S = int(seq_lens.shape[0])
    _check(_lib.pa_prefill(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                           int(block_tables.shape[1]), _ptr(seq_lens), _ptr(query_start), S, T,
                           int(max_query_len), Hq, Hk, d, B, nb, float(softmax_scale),
                           dtype_code(q.dtype), dtype_code(k_cache.dtype), float(k_scale),
                           float(v_scale), _ptr(dev_err), _stream(stream)),
           "pa_prefill")


def pa_cache_write_per_channel(k_new, v_new, k_cache, v_cache, slot_mapping, k_scales, v_scales,
                               dev_err=None, stream=None) -> None:
    """Cache write into an 8-bit pool with per-channel scales (fp32 [Hk, d])."""
    T, Hk, d = (int(x) for x in k_new.shape)
    nb, _, B, _ = (int(x) for x in k_cache.shape)
    _check(_lib.pa_cache_write_per_channel(_ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                                           _ptr(slot_mapping), T, nb, Hk, d, B,
                                           dtype_code(k_new.dtype), dtype_code(k_cache.dtype),
                                           _ptr(k_scales), _ptr(v_scales), _ptr(dev_err),
                                           _stream(stream)),
           "pa_cache_write_per_channel")


def pa_decode_per_channel(out, q, k_cache, v_cache, block_tables, seq_lens, softmax_scale: float,
                          k_scales, v_scales, partition_size: int = 0, max_seq_len: int = 0,
                          workspace=None, dev_err=None, stream=None) -> None:
    """Decode over an 8-bit cache with per-channel scales (partition_size 0:
    single pass; > 0: split-KV with ``workspace``)."""
    S, Hq, d = (int(x) for x in q.shape)
    nb, Hk, B, _ = (int(x) for x in k_cache.shape)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.pa_decode_per_channel(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                      _ptr(block_tables), int(block_tables.shape[1]),
                                      _ptr(seq_lens), S, Hq, Hk, d, B, nb, float(softmax_scale),
                                      dtype_code(q.dtype), dtype_code(k_cache.dtype),
                                      _ptr(k_scales), _ptr(v_scales), int(partition_size),
                                      int(max_seq_len), _ptr(workspace), ws_bytes, _ptr(dev_err),
                                      _stream(stream)),
           "pa_decode_per_channel")


def pa_shared_prefix_workspace_bytes(num_seqs: int, num_q_heads: int, head_dim: int,
                                     max_seq_len: int, prefix_len: int,
                                     partition_size: int) -> int:
    return int(_lib.pa_shared_prefix_workspace_bytes(num_seqs, num_q_heads, head_dim,
                                                     max_seq_len, prefix_len, partition_size))


def pa_decode_shared_prefix(out, q, k_cache, v_cache, block_tables, seq_lens,
                            softmax_scale: float, prefix_len: int, partition_size: int,
                            max_seq_len: int, workspace, dev_err=None, stream=None,
                            k_scale: float = 1.0, v_scale: float = 1.0) -> None:
    """Decode of sequences sharing their first ``prefix_len`` cached tokens
    (the same blocks): the prefix is attended once for all of them."""
    S, Hq, d = (int(x) for x in q.shape)
    nb, Hk, B, _ = (int(x) for x in k_cache.shape)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(_lib.pa_decode_shared_prefix(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                        _ptr(block_tables), int(block_tables.shape[1]),
                                        _ptr(seq_lens), S, Hq, Hk, d, B, nb, float(softmax_scale),
                                        dtype_code(q.dtype), dtype_code(k_cache.dtype),
                                        float(k_scale), float(v_scale), int(prefix_len),
                                        int(partition_size), int(max_seq_len),
                                        _ptr(workspace), ws_bytes, _ptr(dev_err), _stream(stream)),
           "pa_decode_shared_prefix")
