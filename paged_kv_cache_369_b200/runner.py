"""Device-resident decode state and the step that runs the hot path.

``PagedDecode`` uploads one workload (any object with the attributes of
``workload.Workload``): q, this step's new K/V rows, block tables and
lengths, and K/V pools filled with 0xFF (NaN in every cache format) into which
the earlier tokens are written by the library's own slot-mapping and
cache-write kernels.  ``step()`` is one pass of the hot path, all through the
C ABI: slot mapping of the new tokens, cache write, decode (single pass or
split-KV partition + reduce); in the fused modes one pa_decode_append call
whose decode kernel stores the new tokens itself; in cascade mode the write
then pa_decode_shared_prefix.  ``PagedPrefill`` does the same for one
chunked-prefill step.

PyTorch only provides device memory and streams here.
"""

from __future__ import annotations

import math
from typing import Optional

import numpy as np
import torch

from . import (pa_cache_write, pa_cache_write_per_channel, pa_decode, pa_decode_append,
               pa_decode_per_channel, pa_decode_shared_prefix, pa_decode_split_reduce, pa_prefill,
               pa_shared_prefix_workspace_bytes, pa_slot_mapping, pa_split_workspace_bytes,
               pool_torch_dtype)

_TORCH_ACT = {"f16": torch.float16, "bf16": torch.bfloat16}
_UPLOAD_CHUNK_TOKENS = 1 << 16


def _bits_to_device(bits: np.ndarray, act: str, device) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(_TORCH_ACT[act])
    return t.to(device, non_blocking=False)


class PagedDecode:
    """One decode workload resident on a GPU."""

    def __init__(self, w, device: str = "cuda", mode: str = "split", partition_size: int = 512,
                 prefill: bool = True, stream: Optional[torch.cuda.Stream] = None):
        if mode not in ("split", "single", "fused", "fused_single", "cascade"):
            raise ValueError(mode)
        # cascade: sequences sharing a prefix of whole blocks (the workload's
        # shared_prefix_blocks) attend to it once through pa_decode_shared_prefix
        self.prefix_len = getattr(w, "shared_prefix_blocks", 0) * w.block_size
        if mode == "cascade" and self.prefix_len <= 0:
            raise ValueError("cascade mode needs a shared prefix")
        self.per_channel = getattr(w, "k_chan", None) is not None
        if self.per_channel and mode.startswith("fused"):
            raise ValueError("per-channel scales: the cache write is its own call (split / single)")
        self.w = w
        self.device = torch.device(device)
        self.mode = mode
        self.partition_size = partition_size
        self.stream = stream
        S, Hq, Hk, d = w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim
        dev = self.device
        act = _TORCH_ACT[w.act_dtype]
        self.q = _bits_to_device(w.q, w.act_dtype, dev)
        self.k_new = _bits_to_device(w.k_new, w.act_dtype, dev)
        self.v_new = _bits_to_device(w.v_new, w.act_dtype, dev)
        self.block_tables = torch.from_numpy(np.ascontiguousarray(w.block_tables)).to(dev)
        self.seq_lens = torch.from_numpy(np.ascontiguousarray(w.seq_lens)).to(dev)
        pool_dtype = pool_torch_dtype(w.kv_dtype)
        shape = (w.num_blocks, Hk, w.block_size, d)
        self.k_cache = torch.empty(shape, dtype=pool_dtype, device=dev)
        self.v_cache = torch.empty(shape, dtype=pool_dtype, device=dev)
        self.k_cache.view(torch.uint8).fill_(0xFF)
        self.v_cache.view(torch.uint8).fill_(0xFF)
        self.slot_mapping = torch.empty(S, dtype=torch.int64, device=dev)
        # the new token of sequence s (padding -1 for an empty sequence)
        self.new_seq = torch.from_numpy(np.ascontiguousarray(w.new_seq)).to(dev)
        self.out = torch.empty((S, Hq, d), dtype=act, device=dev)
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=dev)
        if self.per_channel:
            self.k_chan = torch.from_numpy(np.ascontiguousarray(w.k_chan, np.float32)).to(dev)
            self.v_chan = torch.from_numpy(np.ascontiguousarray(w.v_chan, np.float32)).to(dev)
        self.max_seq_len = int(w.seq_lens.max()) if S else 0
        nbytes = pa_split_workspace_bytes(S, Hq, d, self.max_seq_len, partition_size)
        if mode == "cascade":
            nbytes = pa_shared_prefix_workspace_bytes(S, Hq, d, self.max_seq_len, self.prefix_len,
                                                      partition_size)
        self.workspace = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
        if prefill:
            self.prefill()

    # -- cache contents that precede the step --------------------------------
    def prefill(self) -> None:
        """Write every earlier token's K/V rows through pa_slot_mapping +
        pa_cache_write, in chunks of tokens."""
        w = self.w
        Tp = int(w.prefill_seq.size)
        dev = self.device
        for lo in range(0, Tp, _UPLOAD_CHUNK_TOKENS):
            hi = min(Tp, lo + _UPLOAD_CHUNK_TOKENS)
            tseq = torch.from_numpy(w.prefill_seq[lo:hi]).to(dev)
            tpos = torch.from_numpy(w.prefill_pos[lo:hi]).to(dev)
            kn = _bits_to_device(w.k_prefill[lo:hi], w.act_dtype, dev)
            vn = _bits_to_device(w.v_prefill[lo:hi], w.act_dtype, dev)
            slots = torch.empty(hi - lo, dtype=torch.int64, device=dev)
            pa_slot_mapping(slots, self.block_tables, self.seq_lens, tseq, tpos, hi - lo,
                            w.num_seqs, w.num_blocks, w.block_size, self.dev_err, self.stream)
            self._cache_write(kn, vn, slots)
        torch.cuda.synchronize(dev)

    def _cache_write(self, kn, vn, slots) -> None:
        w = self.w
        if self.per_channel:
            pa_cache_write_per_channel(kn, vn, self.k_cache, self.v_cache, slots, self.k_chan,
                                       self.v_chan, self.dev_err, self.stream)
        else:
            pa_cache_write(kn, vn, self.k_cache, self.v_cache, slots, w.k_scale, w.v_scale,
                           self.dev_err, self.stream)

    # -- the hot path ----------------------------------------------------------
    def write_new(self) -> None:
        w = self.w
        pa_slot_mapping(self.slot_mapping, self.block_tables, self.seq_lens, self.new_seq, None,
                        w.num_seqs, w.num_seqs, w.num_blocks, w.block_size, self.dev_err,
                        self.stream)
        self._cache_write(self.k_new, self.v_new, self.slot_mapping)

    def attend(self) -> None:
        w = self.w
        if self.per_channel:
            P = 0 if self.mode == "single" else self.partition_size
            pa_decode_per_channel(self.out, self.q, self.k_cache, self.v_cache, self.block_tables,
                                  self.seq_lens, w.softmax_scale, self.k_chan, self.v_chan, P,
                                  self.max_seq_len, self.workspace if P else None, self.dev_err,
                                  self.stream)
            return
        if self.mode == "cascade":
            pa_decode_shared_prefix(self.out, self.q, self.k_cache, self.v_cache,
                                    self.block_tables, self.seq_lens, w.softmax_scale,
                                    self.prefix_len, self.partition_size, self.max_seq_len,
                                    self.workspace, self.dev_err, self.stream, w.k_scale,
                                    w.v_scale)
            return
        if self.mode == "single":
            pa_decode(self.out, self.q, self.k_cache, self.v_cache, self.block_tables,
                      self.seq_lens, w.softmax_scale, w.k_scale, w.v_scale, self.dev_err,
                      self.stream)
        else:
            pa_decode_split_reduce(self.out, self.q, self.k_cache, self.v_cache,
                                   self.block_tables, self.seq_lens, w.softmax_scale,
                                   self.partition_size, self.max_seq_len, self.workspace,
                                   w.k_scale, w.v_scale, self.dev_err, self.stream)

    def fused_step(self) -> None:
        """One decode step through pa_decode_append: the new tokens are stored
        by the attention launch itself."""
        w = self.w
        P = 0 if self.mode == "fused_single" else self.partition_size
        pa_decode_append(self.out, self.q, self.k_new, self.v_new, self.k_cache, self.v_cache,
                         self.block_tables, self.seq_lens, w.softmax_scale, P, self.max_seq_len,
                         self.workspace if P else None, w.k_scale, w.v_scale, self.dev_err,
                         self.stream)

    def step(self) -> None:
        """One decode step: slot mapping, cache write, attention."""
        if self.mode.startswith("fused"):
            self.fused_step()
            return
        self.write_new()
        self.attend()

    def launches_per_step(self) -> int:
        """Kernel launches of one step (the tensor-core route; the CUDA-core
        route of a fused step adds one append launch)."""
        return {"single": 3, "split": 4, "fused": 2, "fused_single": 1, "cascade": 5}[self.mode]

    def error(self) -> int:
        return int(self.dev_err.item())


def default_partition_size(w, config_id=None) -> int:
    """Split-KV partition for a named decode workload: 512 tokens where the
    workload prescribes it (the long-context configuration, config 4); 768
    for the shared-prefix batch (config 5); else 1024.  Measured on B200
    (graph-timed steps) with 512 / 768 / 1024 / 2048: Qwen3-8B shape 96.7 /
    96.1 / 95.1 / 100.0 us; shared-prefix batch, cascade, 214.0 / 211.0 /
    212.6 / 217.0 us."""
    if config_id == 4:
        return 512
    if config_id == 5:
        return 768
    return 1024


def default_mode(config_id=None) -> str:
    """Step for a named decode workload: the fused step (the decode kernel
    stores the new tokens) with split-KV partitions, except for the
    Llama-3-70B shape (config 3), whose even lengths (2048-2560) run best in
    one pass per (sequence, KV head): 52.1 us, against 58.4 / 56.2 / 52.7 us
    with 1024- / 2048- / 2560-token partitions."""
    return "fused_single" if config_id == 3 else "fused"


def algorithmic_decode_bytes(w) -> int:
    """Bytes the attention launch must move: every K/V row read once, q read,
    the output written, block tables and lengths read."""
    S, Hq, d = w.num_seqs, w.num_q_heads, w.head_dim
    return w.kv_bytes_logical() + 2 * S * Hq * d * 2 + int(sum(
        math.ceil(int(L) / w.block_size) for L in w.seq_lens)) * 4 + S * 4


class PagedPrefill:
    """One chunked-prefill step resident on a GPU (any object with the
    attributes of ``workload.ChunkedWorkload``; 16-bit or 8-bit caches).  The
    context tokens are written into 0xFF-poisoned pools at construction;
    ``step()`` appends the chunk's K/V rows (pa_slot_mapping with token
    positions + pa_cache_write) and runs pa_prefill."""

    def __init__(self, w, device: str = "cuda", stream: Optional[torch.cuda.Stream] = None):
        self.w = w
        self.device = torch.device(device)
        self.stream = stream
        dev = self.device
        act = _TORCH_ACT[w.act_dtype]
        T = w.num_tokens
        self.q = _bits_to_device(w.q, w.act_dtype, dev)
        self.k_chunk = _bits_to_device(w.k_chunk, w.act_dtype, dev)
        self.v_chunk = _bits_to_device(w.v_chunk, w.act_dtype, dev)
        self.chunk_seq = torch.from_numpy(np.ascontiguousarray(w.chunk_seq)).to(dev)
        self.chunk_pos = torch.from_numpy(np.ascontiguousarray(w.chunk_pos)).to(dev)
        self.block_tables = torch.from_numpy(np.ascontiguousarray(w.block_tables)).to(dev)
        self.seq_lens = torch.from_numpy(np.ascontiguousarray(w.seq_lens)).to(dev)
        self.query_start = torch.from_numpy(np.ascontiguousarray(w.query_start)).to(dev)
        shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
        self.k_cache = torch.empty(shape, dtype=pool_torch_dtype(w.kv_dtype), device=dev)
        self.v_cache = torch.empty(shape, dtype=pool_torch_dtype(w.kv_dtype), device=dev)
        self.k_cache.view(torch.uint8).fill_(0xFF)
        self.v_cache.view(torch.uint8).fill_(0xFF)
        self.slots = torch.empty(max(T, 1), dtype=torch.int64, device=dev)
        self.out = torch.empty((T, w.num_q_heads, w.head_dim), dtype=act, device=dev)
        self.dev_err = torch.zeros(1, dtype=torch.int32, device=dev)
        self._write(w.ctx_seq, w.ctx_pos, w.k_ctx, w.v_ctx)
        torch.cuda.synchronize(dev)

    def _write(self, seq, pos, kr, vr) -> None:
        w, dev = self.w, self.device
        for lo in range(0, int(seq.size), _UPLOAD_CHUNK_TOKENS):
            hi = min(int(seq.size), lo + _UPLOAD_CHUNK_TOKENS)
            tseq = torch.from_numpy(seq[lo:hi]).to(dev)
            tpos = torch.from_numpy(pos[lo:hi]).to(dev)
            kn = _bits_to_device(kr[lo:hi], w.act_dtype, dev)
            vn = _bits_to_device(vr[lo:hi], w.act_dtype, dev)
            slots = torch.empty(hi - lo, dtype=torch.int64, device=dev)
            pa_slot_mapping(slots, self.block_tables, self.seq_lens, tseq, tpos, hi - lo,
                            w.num_seqs, w.num_blocks, w.block_size, self.dev_err, self.stream)
            pa_cache_write(kn, vn, self.k_cache, self.v_cache, slots, w.k_scale, w.v_scale,
                           self.dev_err, self.stream)

    def write_chunk(self) -> None:
        w = self.w
        T = w.num_tokens
        if T == 0:
            return
        pa_slot_mapping(self.slots, self.block_tables, self.seq_lens, self.chunk_seq,
                        self.chunk_pos, T, w.num_seqs, w.num_blocks, w.block_size, self.dev_err,
                        self.stream)
        pa_cache_write(self.k_chunk, self.v_chunk, self.k_cache, self.v_cache, self.slots,
                       w.k_scale, w.v_scale, self.dev_err, self.stream)

    def attend(self) -> None:
        w = self.w
        pa_prefill(self.out, self.q, self.k_cache, self.v_cache, self.block_tables, self.seq_lens,
                   self.query_start, w.max_query_len, w.softmax_scale, self.dev_err, self.stream,
                   w.k_scale, w.v_scale)

    def step(self) -> None:
        self.write_chunk()
        self.attend()

    def error(self) -> int:
        return int(self.dev_err.item())


def algorithmic_cascade_bytes(w) -> int:
    """Bytes the shared-prefix decode must move: the shared prefix's K/V once,
    every sequence's tail K/V once, q read, the output written, tables and
    lengths read."""
    S, Hq, Hk, d = w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim
    prefix = w.shared_prefix_blocks * w.block_size
    per_tok = Hk * 2 * d * w.kv_elem_bytes()
    tails = int((w.seq_lens.astype(np.int64) - prefix).clip(min=0).sum())
    return (prefix + tails) * per_tok + 2 * S * Hq * d * 2 + int(sum(
        math.ceil(int(L) / w.block_size) for L in w.seq_lens)) * 4 + S * 4
