"""Seeded synthetic paged-KV decode workloads.

This module only *creates inputs*: sequence lengths, a shuffled physical block
pool, per-sequence block tables (with a shared, reference-counted prefix where
asked), query / key / value values drawn from N(0, 1) and rounded to the
activation dtype, and the per-tensor fp8 scales.  It holds none of the
method's arithmetic: no slot addressing, no cache write, no quantisation, no
attention.  Both the CUDA path and the CPU oracle consume what it returns, each
doing the method's steps on its own.

Values are returned as raw 16-bit patterns (``np.uint16``) in the activation
dtype ("f16" = IEEE binary16, "bf16" = bfloat16) so that neither consumer
depends on the other's numeric types.

The five named workloads follow the decode configurations that the pages'
problem statement is built around:

1. tiny: GQA 4/2, d=64, lengths [10, 45, 20, 33], f16, a 32-block pool;
2. Qwen3-8B-shaped: 64 sequences, 32/8 heads, d=128, lengths U[512, 4096], bf16;
3. Llama-3-70B-shaped: 32 sequences, 64/8 heads, lengths U[2048, 2560], bf16;
4. long context: 8 x 32768 tokens, 64/8 heads, fp8-E4M3 KV with a per-tensor
   scale, bf16 query;
5. continuous batching: 256 sequences, MHA 32/32, all sharing one 1024-token
   prefix (same physical blocks, refcount 256) plus private lognormal tails of
   mean 300 tokens clipped to [1, 2048], f16.

Block size is 16 tokens throughout ("Transformer 推理优化：KV Cache、PagedAttention
与 vLLM", §3.2).  The pool holds the blocks in use plus 10 % free blocks; the
physical ids are a seeded Fisher-Yates permutation of the pool, handed out in
sequence order, so logically adjacent blocks sit far apart in memory.
"""

from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import numpy as np
import torch

SEED_BASE = 369000
BLOCK_SIZE = 16
_CHUNK = 1 << 24  # values drawn per chunk when filling large K/V arrays


@dataclasses.dataclass
class Workload:
    """One decode step's inputs plus the cache contents that precede it."""

    name: str
    seed: int
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    act_dtype: str  # dtype of q, of the new K/V rows and of the output
    kv_dtype: str  # dtype of the cache pools: "f16" | "bf16" | "e4m3" | "e5m2" | "int8"
    seq_lens: np.ndarray  # int32 [S]; counts the token written by this step
    block_tables: np.ndarray  # int32 [S, max_blocks_per_seq]
    refcount: np.ndarray  # int32 [num_blocks]: tables referencing each block
    q: np.ndarray  # uint16 [S, Hq, d]
    # tokens already in the cache before this step (positions < seq_len - 1)
    prefill_seq: np.ndarray  # int32 [Tp]
    prefill_pos: np.ndarray  # int32 [Tp]
    k_prefill: np.ndarray  # uint16 [Tp, Hk, d]
    v_prefill: np.ndarray  # uint16 [Tp, Hk, d]
    # this step's new token of every sequence, at position seq_len - 1
    k_new: np.ndarray  # uint16 [S, Hk, d]
    v_new: np.ndarray  # uint16 [S, Hk, d]
    k_scale: float  # fp32 value; 1.0 unless the cache is 8-bit
    v_scale: float
    free_blocks: np.ndarray  # int32: physical ids no table references
    shared_prefix_blocks: int = 0
    # per-channel scales of an 8-bit cache, fp32 [Hk, d] (None: per tensor)
    k_chan: Optional[np.ndarray] = None
    v_chan: Optional[np.ndarray] = None

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_lens.max()) if self.num_seqs else 0

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def new_seq(self) -> np.ndarray:
        """Sequence index of each new token (one per sequence); -1 (padding)
        for an empty sequence, which has no token to write."""
        idx = np.arange(self.num_seqs, dtype=np.int32)
        return np.where(self.seq_lens > 0, idx, -1).astype(np.int32)

    @property
    def new_pos(self) -> np.ndarray:
        """Position of each new token: the last one of its sequence."""
        return (self.seq_lens - 1).astype(np.int32)

    def kv_elem_bytes(self) -> int:
        return 1 if self.kv_dtype in EIGHT_BIT else 2

    def act_elem_bytes(self) -> int:
        return 2

    def kv_bytes_logical(self) -> int:
        """K+V bytes one decode pass reads: sum_s L_s * Hk * 2 * d * b_kv."""
        return int(self.seq_lens.astype(np.int64).sum()) * self.num_kv_heads * 2 * self.head_dim * self.kv_elem_bytes()

    def step_bytes(self) -> int:
        """Algorithmic bytes of one step: K/V read once, q read, out written,
        block tables and lengths read, and the new K/V rows written once
        (read as activations, written into the pools)."""
        S, Hq, Hk, d = self.num_seqs, self.num_q_heads, self.num_kv_heads, self.head_dim
        qo = 2 * S * Hq * d * self.act_elem_bytes()
        tables = self.block_tables.size * 4 + S * 4
        new_rows = S * Hk * d * 2 * (self.act_elem_bytes() + self.kv_elem_bytes())
        return self.kv_bytes_logical() + qo + tables + new_rows

    def pool_elems(self) -> int:
        return self.num_blocks * self.num_kv_heads * self.block_size * self.head_dim


# ----------------------------------------------------------------------------
# value drawing
# ----------------------------------------------------------------------------

def f32_to_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round fp32 values to f16 / bf16 (round to nearest even) and return the
    16-bit patterns.  This is input creation, done by torch's converters."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "f16":
        return t.to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    if dtype == "bf16":
        return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    raise ValueError(f"unsupported activation dtype {dtype!r}")


def bits_to_f32(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Widen 16-bit patterns back to fp32 (exact)."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    if dtype == "f16":
        return t.view(torch.float16).float().numpy()
    if dtype == "bf16":
        return t.view(torch.bfloat16).float().numpy()
    raise ValueError(dtype)


def draw_normal_bits(rng: np.random.Generator, shape, dtype: str) -> np.ndarray:
    """N(0, 1) values drawn in fp32 and rounded to ``dtype``, filled in chunks."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    for lo in range(0, n, _CHUNK):
        hi = min(n, lo + _CHUNK)
        out[lo:hi] = f32_to_bits(rng.standard_normal(hi - lo, dtype=np.float32), dtype)
    return out.reshape(shape)


def amax_of_bits(*arrays: np.ndarray, dtype: str) -> float:
    m = 0.0
    for a in arrays:
        flat = a.reshape(-1)
        for lo in range(0, flat.size, _CHUNK):
            m = max(m, float(np.abs(bits_to_f32(flat[lo:lo + _CHUNK], dtype)).max(initial=0.0)))
    return m


EIGHT_BIT = ("e4m3", "e5m2", "int8")

# largest code magnitude of each 8-bit cache format: E4M3 448 and E5M2 57344
# ("大语言模型推理引擎深度剖析", §4.2), symmetric INT8 127
CODE_MAX = {"e4m3": 448.0, "e5m2": 57344.0, "int8": 127.0}


def per_tensor_e4m3_scale(amax: float) -> float:
    """Per-tensor fp8 scale amax / 448 as an fp32 value (448 is the E4M3
    maximum: "大语言模型推理引擎深度剖析", §4.2).  A zero amax gives scale 1."""
    return per_tensor_scale(amax, "e4m3")


def per_channel_scales(kv_dtype: str, *arrays: np.ndarray, dtype: str) -> np.ndarray:
    """Scale of every (KV head, channel): the channel's amax over all tokens of
    the given [T, Hk, d] rows / (largest code), fp32 [Hk, d]; zero amax gives 1
    (the fifth page's §4.3 quantises each channel of K / V separately)."""
    amax = None
    for a in arrays:
        for lo in range(0, a.shape[0], max(1, _CHUNK // max(1, a.shape[1] * a.shape[2]))):
            hi = min(a.shape[0], lo + max(1, _CHUNK // max(1, a.shape[1] * a.shape[2])))
            m = np.abs(bits_to_f32(a[lo:hi], dtype)).max(axis=0, initial=0.0)
            amax = m if amax is None else np.maximum(amax, m)
    amax = amax.astype(np.float32)
    sc = amax / np.float32(CODE_MAX[kv_dtype])
    return np.where(amax > 0, sc, np.float32(1.0)).astype(np.float32)


def per_tensor_scale(amax: float, kv_dtype: str) -> float:
    """Per-tensor scale amax / (largest code) of an 8-bit cache format, as an
    fp32 value; a zero amax gives scale 1."""
    if amax <= 0.0:
        return 1.0
    return float(np.float32(amax) / np.float32(CODE_MAX[kv_dtype]))


# ----------------------------------------------------------------------------
# block pool and tables
# ----------------------------------------------------------------------------

def blocks_needed(length: int, block_size: int) -> int:
    return -(-int(length) // block_size)


def build(
    name: str,
    seed: int,
    seq_lens: Sequence[int],
    num_q_heads: int,
    num_kv_heads: int,
    head_dim: int,
    act_dtype: str,
    kv_dtype: str,
    block_size: int = BLOCK_SIZE,
    num_blocks: Optional[int] = None,
    pool_slack: float = 0.10,
    shared_prefix_tokens: int = 0,
    extra_table_cols: int = 0,
    draw_kv: bool = True,
    channel_scales: bool = False,
) -> Workload:
    """Draw one workload.

    ``shared_prefix_tokens`` (a multiple of ``block_size``) makes every table
    start with the same physical blocks.  ``extra_table_cols`` appends unused
    table columns (filled with a free block id, so an over-read lands on
    poisoned memory instead of outside the pool).  ``draw_kv=False`` skips the
    prefill values (shape-only workloads for host-side tests).
    ``channel_scales`` gives an 8-bit cache one scale per (KV head, channel).
    """
    rng = np.random.default_rng(seed)
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    S = int(seq_lens.size)
    if shared_prefix_tokens % block_size:
        raise ValueError("shared prefix must be block aligned")
    if seq_lens.size and int(seq_lens.min()) < 0:
        raise ValueError("negative sequence length")
    if shared_prefix_tokens and S and int(seq_lens.min()) <= shared_prefix_tokens:
        raise ValueError("every sequence must extend past the shared prefix")
    nprefix = shared_prefix_tokens // block_size
    nblk = [blocks_needed(L, block_size) for L in seq_lens]
    private = [b - nprefix for b in nblk] if nprefix else nblk
    used = nprefix + int(sum(private))
    if num_blocks is None:
        num_blocks = max(used + 1, int(math.ceil(used * (1.0 + pool_slack))))
    if num_blocks < used:
        raise ValueError("pool too small")
    perm = rng.permutation(num_blocks).astype(np.int32)  # Fisher-Yates shuffle
    mbs = max(max(nblk, default=0), 1) + extra_table_cols
    cursor = 0
    prefix_ids = perm[cursor:cursor + nprefix]
    cursor += nprefix
    tables = np.empty((S, mbs), dtype=np.int32)
    refcount = np.zeros(num_blocks, dtype=np.int32)
    for s in range(S):
        own = perm[cursor:cursor + private[s]]
        cursor += private[s]
        row = np.concatenate([prefix_ids, own]) if nprefix else own
        tables[s, :row.size] = row
        refcount[row] += 1
        tables[s, row.size:] = -1
    free = perm[cursor:].copy()
    pad = int(free[0]) if free.size else 0
    tables[tables < 0] = pad

    q = draw_normal_bits(rng, (S, num_q_heads, head_dim), act_dtype)
    k_new = draw_normal_bits(rng, (S, num_kv_heads, head_dim), act_dtype)
    v_new = draw_normal_bits(rng, (S, num_kv_heads, head_dim), act_dtype)

    # tokens present before this step: the shared prefix once (through the
    # first table), then every sequence's own tokens up to position L - 2
    pseq: List[np.ndarray] = []
    ppos: List[np.ndarray] = []
    if nprefix and S:
        pseq.append(np.zeros(shared_prefix_tokens, dtype=np.int32))
        ppos.append(np.arange(shared_prefix_tokens, dtype=np.int32))
    for s in range(S):
        lo = shared_prefix_tokens if nprefix else 0
        hi = int(seq_lens[s]) - 1
        if hi > lo:
            pseq.append(np.full(hi - lo, s, dtype=np.int32))
            ppos.append(np.arange(lo, hi, dtype=np.int32))
    prefill_seq = np.concatenate(pseq) if pseq else np.zeros(0, np.int32)
    prefill_pos = np.concatenate(ppos) if ppos else np.zeros(0, np.int32)
    Tp = int(prefill_seq.size)
    if draw_kv:
        k_prefill = draw_normal_bits(rng, (Tp, num_kv_heads, head_dim), act_dtype)
        v_prefill = draw_normal_bits(rng, (Tp, num_kv_heads, head_dim), act_dtype)
    else:
        k_prefill = np.zeros((0, num_kv_heads, head_dim), np.uint16)
        v_prefill = np.zeros((0, num_kv_heads, head_dim), np.uint16)
        prefill_seq = prefill_seq[:0]
        prefill_pos = prefill_pos[:0]

    k_scale = v_scale = 1.0
    k_chan = v_chan = None
    if kv_dtype in EIGHT_BIT:
        k_scale = per_tensor_scale(amax_of_bits(k_prefill, k_new, dtype=act_dtype), kv_dtype)
        v_scale = per_tensor_scale(amax_of_bits(v_prefill, v_new, dtype=act_dtype), kv_dtype)
        if channel_scales:
            k_chan = per_channel_scales(kv_dtype, k_prefill, k_new, dtype=act_dtype)
            v_chan = per_channel_scales(kv_dtype, v_prefill, v_new, dtype=act_dtype)
    elif kv_dtype != act_dtype:
        raise ValueError("a 16-bit cache must have the activation dtype")
    elif channel_scales:
        raise ValueError("per-channel scales need an 8-bit cache")

    return Workload(
        name=name, seed=seed, num_seqs=S, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
        head_dim=head_dim, block_size=block_size, num_blocks=int(num_blocks),
        act_dtype=act_dtype, kv_dtype=kv_dtype, seq_lens=seq_lens, block_tables=tables,
        refcount=refcount, q=q, prefill_seq=prefill_seq, prefill_pos=prefill_pos,
        k_prefill=k_prefill, v_prefill=v_prefill, k_new=k_new, v_new=v_new,
        k_scale=k_scale, v_scale=v_scale, free_blocks=free, shared_prefix_blocks=nprefix,
        k_chan=k_chan, v_chan=v_chan,
    )


# ----------------------------------------------------------------------------
# the five named decode workloads
# ----------------------------------------------------------------------------

CONFIG_NAMES = {
    1: "tiny paged decode: GQA 4/2, d64, lens [10,45,20,33], f16, 32-block pool",
    2: "Qwen3-8B-shaped decode: 64 seqs, 32/8 heads, d128, lens U[512,4096], bf16",
    3: "Llama-3-70B-shaped decode: 32 seqs, 64/8 heads, d128, lens U[2048,2560], bf16",
    4: "long-context fp8 KV: 8 x 32768, 64/8 heads, d128, E4M3 per-tensor scale, bf16 q, split 512",
    5: "continuous batching: 256 seqs, MHA 32/32, d128, shared 1024-token prefix + lognormal tails, f16",
}


def config_seq_lens(cfg: int, rng: np.random.Generator) -> np.ndarray:
    if cfg == 1:
        return np.array([10, 45, 20, 33], dtype=np.int32)
    if cfg == 2:
        return rng.integers(512, 4096, size=64, endpoint=True).astype(np.int32)
    if cfg == 3:
        return rng.integers(2048, 2560, size=32, endpoint=True).astype(np.int32)
    if cfg == 4:
        return np.full(8, 32768, dtype=np.int32)
    if cfg == 5:
        sigma = 1.0
        mu = math.log(300.0) - sigma * sigma / 2.0  # pre-clip mean 300
        tails = np.rint(rng.lognormal(mu, sigma, size=256))
        tails = np.clip(tails, 1, 2048).astype(np.int32)
        return (1024 + tails).astype(np.int32)
    raise ValueError(f"unknown config {cfg}")


def config(cfg: int, draw_kv: bool = True, kv_dtype: Optional[str] = None,
           channel_scales: bool = False) -> Workload:
    """The named decode workload ``cfg`` (1..5), seeded with 369000 + cfg.
    ``kv_dtype`` replaces the configuration's cache format by an 8-bit one
    ("e4m3", "e5m2", "int8"; same shapes, lengths and seed);
    ``channel_scales`` gives an 8-bit cache per-channel scales."""
    seed = SEED_BASE + cfg
    lens = config_seq_lens(cfg, np.random.default_rng([seed, 1]))
    name = CONFIG_NAMES[cfg]
    if kv_dtype is not None and kv_dtype not in EIGHT_BIT:
        raise ValueError("the cache format can be replaced by an 8-bit one only")

    def kv(default):
        return kv_dtype or default

    if kv_dtype is not None or channel_scales:
        name = f"{name} [{kv_dtype or 'e4m3'} KV, per-{'channel' if channel_scales else 'tensor'} scale]"
    cs = dict(channel_scales=True) if channel_scales else {}
    if cfg == 1:
        return build(name, seed, lens, 4, 2, 64, "f16", kv("f16"), num_blocks=32, draw_kv=draw_kv,
                     **cs)
    if cfg == 2:
        return build(name, seed, lens, 32, 8, 128, "bf16", kv("bf16"), draw_kv=draw_kv, **cs)
    if cfg == 3:
        return build(name, seed, lens, 64, 8, 128, "bf16", kv("bf16"), draw_kv=draw_kv, **cs)
    if cfg == 4:
        return build(name, seed, lens, 64, 8, 128, "bf16", kv("e4m3"), draw_kv=draw_kv, **cs)
    if cfg == 5:
        return build(name, seed, lens, 32, 32, 128, "f16", kv("f16"), shared_prefix_tokens=1024,
                     draw_kv=draw_kv, **cs)
    raise ValueError(cfg)


def poison_byte() -> int:
    """Fill byte for pools before any write: 0xFF makes every f16 / bf16 pair
    and every E4M3 byte a NaN, so any read of an unwritten slot shows up."""
    return 0xFF


# ----------------------------------------------------------------------------
# chunked prefill: several new query tokens per sequence
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class ChunkedWorkload:
    """One chunked-prefill step: every sequence has ``context_lens[s]`` tokens
    in the cache and appends a chunk of ``chunk_lens[s]`` tokens, whose
    queries then attend causally over the context and the chunk."""

    name: str
    seed: int
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    act_dtype: str
    kv_dtype: str
    seq_lens: np.ndarray  # int32 [S]: context + chunk
    query_start: np.ndarray  # int32 [S + 1]: chunk rows of sequence s in q / out
    block_tables: np.ndarray  # int32 [S, max_blocks_per_seq]
    q: np.ndarray  # uint16 [T, Hq, d], T = total chunk tokens
    ctx_seq: np.ndarray  # int32 [Tc]: context tokens (already cached)
    ctx_pos: np.ndarray
    k_ctx: np.ndarray  # uint16 [Tc, Hk, d]
    v_ctx: np.ndarray
    chunk_seq: np.ndarray  # int32 [T]: this chunk's tokens, in q row order
    chunk_pos: np.ndarray
    k_chunk: np.ndarray  # uint16 [T, Hk, d]
    v_chunk: np.ndarray
    k_scale: float
    v_scale: float
    free_blocks: np.ndarray

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def num_tokens(self) -> int:
        return int(self.query_start[-1])

    @property
    def chunk_lens(self) -> np.ndarray:
        return np.diff(self.query_start).astype(np.int32)

    @property
    def max_query_len(self) -> int:
        return int(self.chunk_lens.max()) if self.num_seqs else 0

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    def attended_pairs(self) -> int:
        """(query token, key) pairs under the causal mask, per query head."""
        n = self.chunk_lens.astype(np.int64)
        ctx = self.seq_lens.astype(np.int64) - n
        return int((n * ctx + n * (n + 1) // 2).sum())

    def flops(self) -> int:
        """Useful multiply-adds x 2 of q.K and P.V under the causal mask."""
        return 4 * self.head_dim * self.num_q_heads * self.attended_pairs()


def build_chunked(
    name: str,
    seed: int,
    context_lens: Sequence[int],
    chunk_lens: Sequence[int],
    num_q_heads: int,
    num_kv_heads: int,
    head_dim: int,
    act_dtype: str,
    kv_dtype: str,
    block_size: int = BLOCK_SIZE,
    num_blocks: Optional[int] = None,
    pool_slack: float = 0.10,
    extra_table_cols: int = 0,
) -> ChunkedWorkload:
    """Draw a chunked-prefill step: tables over a shuffled pool (as ``build``),
    context K/V rows, the chunk's q and K/V rows, all N(0, 1) rounded to the
    activation dtype."""
    rng = np.random.default_rng(seed)
    ctx = np.asarray(context_lens, dtype=np.int32)
    chk = np.asarray(chunk_lens, dtype=np.int32)
    if ctx.shape != chk.shape or (ctx.size and (int(ctx.min()) < 0 or int(chk.min()) < 0)):
        raise ValueError("context and chunk lengths must be non-negative and paired")
    S = int(ctx.size)
    lens = (ctx + chk).astype(np.int32)
    nblk = [blocks_needed(L, block_size) for L in lens]
    used = int(sum(nblk))
    if num_blocks is None:
        num_blocks = max(used + 1, int(math.ceil(used * (1.0 + pool_slack))))
    if num_blocks < used:
        raise ValueError("pool too small")
    perm = rng.permutation(num_blocks).astype(np.int32)
    mbs = max(max(nblk, default=0), 1) + extra_table_cols
    tables = np.empty((S, mbs), dtype=np.int32)
    cursor = 0
    for s in range(S):
        tables[s, :nblk[s]] = perm[cursor:cursor + nblk[s]]
        cursor += nblk[s]
    free = perm[cursor:].copy()
    pad = int(free[0]) if free.size else 0
    for s in range(S):
        tables[s, nblk[s]:] = pad
    query_start = np.zeros(S + 1, dtype=np.int32)
    query_start[1:] = np.cumsum(chk)
    T = int(query_start[-1])
    q = draw_normal_bits(rng, (T, num_q_heads, head_dim), act_dtype)
    chunk_seq = np.repeat(np.arange(S, dtype=np.int32), chk)
    chunk_pos = np.concatenate([np.arange(c, c + n, dtype=np.int32) for c, n in zip(ctx, chk)]) \
        if S else np.zeros(0, np.int32)
    k_chunk = draw_normal_bits(rng, (T, num_kv_heads, head_dim), act_dtype)
    v_chunk = draw_normal_bits(rng, (T, num_kv_heads, head_dim), act_dtype)
    ctx_seq = np.repeat(np.arange(S, dtype=np.int32), ctx)
    ctx_pos = np.concatenate([np.arange(0, c, dtype=np.int32) for c in ctx]) \
        if S else np.zeros(0, np.int32)
    Tc = int(ctx_seq.size)
    k_ctx = draw_normal_bits(rng, (Tc, num_kv_heads, head_dim), act_dtype)
    v_ctx = draw_normal_bits(rng, (Tc, num_kv_heads, head_dim), act_dtype)
    k_scale = v_scale = 1.0
    if kv_dtype in EIGHT_BIT:
        k_scale = per_tensor_scale(amax_of_bits(k_ctx, k_chunk, dtype=act_dtype), kv_dtype)
        v_scale = per_tensor_scale(amax_of_bits(v_ctx, v_chunk, dtype=act_dtype), kv_dtype)
    elif kv_dtype != act_dtype:
        raise ValueError("a 16-bit cache must have the activation dtype")
    return ChunkedWorkload(
        name=name, seed=seed, num_seqs=S, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
        head_dim=head_dim, block_size=block_size, num_blocks=int(num_blocks),
        act_dtype=act_dtype, kv_dtype=kv_dtype, seq_lens=lens, query_start=query_start,
        block_tables=tables, q=q, ctx_seq=ctx_seq, ctx_pos=ctx_pos, k_ctx=k_ctx, v_ctx=v_ctx,
        chunk_seq=chunk_seq, chunk_pos=chunk_pos, k_chunk=k_chunk, v_chunk=v_chunk,
        k_scale=k_scale, v_scale=v_scale, free_blocks=free,
    )


PREFILL_NAMES = {
    1: "chunked prefill, Qwen3-8B-shaped: 16 seqs x 512-token chunk after contexts U[0,3584], "
       "32/8 heads, d128, bf16",
    2: "chunked prefill, Llama-3-70B-shaped: 8 seqs x 512-token chunk after contexts U[1536,2048], "
       "64/8 heads, d128, bf16",
}


def prefill_config(cfg: int, kv_dtype: Optional[str] = None) -> ChunkedWorkload:
    """Named chunked-prefill workloads: 512-token chunks (the chunk size the
    pages give) on the decode configurations' model shapes; ``kv_dtype``
    swaps in an 8-bit cache (per-tensor scales)."""
    seed = SEED_BASE + 100 + cfg
    rng = np.random.default_rng([seed, 1])
    kv = kv_dtype or "bf16"
    if cfg == 1:
        ctx = rng.integers(0, 3584, size=16, endpoint=True)
        name = PREFILL_NAMES[1] if kv == "bf16" else f"{PREFILL_NAMES[1]}, {kv} cache"
        return build_chunked(name, seed, ctx, [512] * 16, 32, 8, 128, "bf16", kv)
    if cfg == 2:
        ctx = rng.integers(1536, 2048, size=8, endpoint=True)
        name = PREFILL_NAMES[2] if kv == "bf16" else f"{PREFILL_NAMES[2]}, {kv} cache"
        return build_chunked(name, seed, ctx, [512] * 8, 64, 8, 128, "bf16", kv)
    raise ValueError(f"unknown prefill config {cfg}")
