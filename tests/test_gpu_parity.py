"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bars:
  - cache pools (slot mapping + cache write): bit-exact, untouched bytes included;
  - attention outputs: max-abs error <= 1e-2 and relative L2 error <= 2e-3
    against the fp64 oracle, over the whole output (small cases) or over the
    sampled (sequence, head) rows (full-size workloads); the fp8 oracle
    dequantises the identical E4M3 codes (its own pool, bit-equal to the GPU's);
  - split partials: the partition log-sum-exp and normalised output against
    the oracle's, same bars.
"""

import math
import os

import numpy as np
import pytest
import torch

import oracle
import workload

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
REL_L2 = 2e-3


def _pa():
    import paged_kv_cache_369_b200 as pa
    from paged_kv_cache_369_b200.runner import PagedDecode

    return pa, PagedDecode


def _to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def assert_close(got: np.ndarray, ref: np.ndarray, what: str):
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    max_abs = float(err.max()) if err.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(got - ref)) / denom if denom > 0 else float(np.linalg.norm(got))
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    return max_abs, rel


def pool_bytes(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.uint8).cpu().numpy()


def check_pools(dec, kc, vc):
    assert np.array_equal(pool_bytes(dec.k_cache), kc.view(np.uint8).reshape(pool_bytes(dec.k_cache).shape))
    assert np.array_equal(pool_bytes(dec.v_cache), vc.view(np.uint8).reshape(pool_bytes(dec.v_cache).shape))


GUARD = 4096  # bytes of poison on each side of a guarded buffer (keeps 256-byte alignment)
GUARD_BYTE = 0xA5


def guarded_like(t: torch.Tensor):
    """A tensor shaped and typed like ``t`` inside a larger buffer whose
    GUARD bytes before and after it are filled with GUARD_BYTE; returns
    (buffer, view).  A kernel that writes past either end of the view changes
    the guard bytes."""
    n = t.numel() * t.element_size()
    buf = torch.full((n + 2 * GUARD,), GUARD_BYTE, dtype=torch.uint8, device=t.device)
    view = buf[GUARD:GUARD + n].view(t.dtype).view(t.shape)
    view.copy_(t)
    return buf, view


def check_guards(buf: torch.Tensor, what: str):
    head, tail = buf[:GUARD].cpu().numpy(), buf[-GUARD:].cpu().numpy()
    assert (head == GUARD_BYTE).all(), f"{what}: write before the buffer"
    assert (tail == GUARD_BYTE).all(), f"{what}: write past the end of the buffer"


def sample_pairs(w, n, seed=0):
    rng = np.random.default_rng(seed)
    S, Hq = w.num_seqs, w.num_q_heads
    longest, shortest = int(np.argmax(w.seq_lens)), int(np.argmin(w.seq_lens))
    pairs = {(longest, 0), (longest, Hq - 1), (shortest, Hq // 2), (S - 1, Hq - 1), (0, 0)}
    while len(pairs) < min(n, S * Hq):
        pairs.add((int(rng.integers(S)), int(rng.integers(Hq))))
    return np.array(sorted(pairs), dtype=np.int32)


# ---------------------------------------------------------------------------
# small cases: everything compared
# ---------------------------------------------------------------------------

SMALL = [
    # (Hq, Hk, d, act, kv, lens, prefix)
    (4, 2, 64, "f16", "f16", [10, 45, 20, 33], 0),
    (32, 8, 128, "bf16", "bf16", [1, 15, 16, 17, 31, 32, 33, 100, 513, 700], 0),
    (64, 8, 128, "bf16", "bf16", [2048, 1, 2100, 16], 0),
    (8, 8, 128, "f16", "f16", [1040, 1030, 1100], 1024),
    (64, 8, 128, "bf16", "e4m3", [600, 1, 17, 1024], 0),
    (16, 2, 64, "f16", "e4m3", [3, 90, 16], 0),
    (6, 2, 64, "bf16", "bf16", [5, 70, 18], 0),     # g = 3 (padded to 4)
    (10, 2, 128, "f16", "f16", [40, 9], 0),         # g = 5 (padded to 8)
    (32, 2, 128, "bf16", "bf16", [300, 77], 0),     # g = 16 (two head groups)
    (12, 2, 64, "bf16", "e4m3", [129, 64], 0),      # g = 6
    (2, 2, 64, "f16", "f16", [0, 1, 0, 5], 0),      # empty sequences
    (64, 8, 128, "bf16", "e5m2", [600, 1, 17, 1024], 0),
    (8, 8, 128, "f16", "e5m2", [100, 1100, 33], 0),  # MHA, E5M2
    (32, 8, 128, "f16", "int8", [300, 16, 33, 1], 0),
    (64, 4, 128, "bf16", "int8", [700, 129], 0),    # g = 16, INT8
    (16, 2, 64, "bf16", "int8", [3, 90, 16], 0),    # d = 64: CUDA-core kernel
    (4, 2, 64, "f16", "e5m2", [45, 20], 0),
]


@pytest.fixture(params=["auto", "simt"])
def kernel_choice(request, monkeypatch):
    """Run a test with the default decode kernel (tensor cores wherever the
    shape allows) and with the CUDA-core kernel forced."""
    if request.param == "simt":
        monkeypatch.setenv("PA369_DECODE_KERNEL", "simt")
    else:
        monkeypatch.delenv("PA369_DECODE_KERNEL", raising=False)
    return request.param


@pytest.mark.parametrize("mode,P", [("single", 512), ("split", 512), ("split", 16), ("split", 64),
                                    ("fused", 512), ("fused", 16), ("fused_single", 512)])
@pytest.mark.parametrize("case", range(len(SMALL)))
def test_small_full_parity(case, mode, P, kernel_choice):
    pa, PagedDecode = _pa()
    Hq, Hk, d, act, kv, lens, prefix = SMALL[case]
    w = workload.build(f"small{case}", 1000 + case, lens, Hq, Hk, d, act, kv,
                       shared_prefix_tokens=prefix, extra_table_cols=2)
    dec = PagedDecode(w, mode=mode, partition_size=P)
    # out and the split workspace sit between poisoned guard bands
    out_buf, dec.out = guarded_like(dec.out)
    ws_buf, dec.workspace = guarded_like(dec.workspace)
    dec.step()
    torch.cuda.synchronize()
    assert dec.error() == 0
    check_guards(out_buf, "out")
    check_guards(ws_buf, "workspace")
    kc, vc = oracle.caches_for(w)
    check_pools(dec, kc, vc)
    ref = oracle.decode_for(w, kc, vc)
    got = _to_f64(dec.out)
    assert_close(got, ref, f"case {case} {mode} P={P} kernel={kernel_choice}")
    # empty sequences give exact zeros
    for s in range(w.num_seqs):
        if w.seq_lens[s] == 0:
            assert not got[s].any()


@pytest.mark.parametrize("chain", ["2", "3"])
@pytest.mark.parametrize("mode", ["split", "fused"])
@pytest.mark.parametrize("case", [c for c in range(len(SMALL)) if max(SMALL[c][5]) > 16 * 16])
def test_chained_partitions_parity(case, mode, chain, monkeypatch):
    """Long split contexts (16 or more partitions) run with each warp taking
    several consecutive partitions in a row and writing each one's partial as
    it crosses into the next; PA369_DECODE_CHAIN forces 2 or 3 a warp, so
    that the boundaries fall inside a warp's run, at sequence ends and in a
    CTA's second warp.  16-token partitions."""
    monkeypatch.setenv("PA369_DECODE_CHAIN", chain)
    pa, PagedDecode = _pa()
    Hq, Hk, d, act, kv, lens, prefix = SMALL[case]
    w = workload.build(f"small{case}", 1000 + case, lens, Hq, Hk, d, act, kv,
                       shared_prefix_tokens=prefix, extra_table_cols=2)
    dec = PagedDecode(w, mode=mode, partition_size=16)
    out_buf, dec.out = guarded_like(dec.out)
    ws_buf, dec.workspace = guarded_like(dec.workspace)
    dec.step()
    torch.cuda.synchronize()
    assert dec.error() == 0
    check_guards(out_buf, "out")
    check_guards(ws_buf, "workspace")
    kc, vc = oracle.caches_for(w)
    check_pools(dec, kc, vc)
    ref = oracle.decode_for(w, kc, vc)
    assert_close(_to_f64(dec.out), ref, f"case {case} {mode} chain={chain}")


PER_CHANNEL = [
    # (Hq, Hk, d, act, kv, lens)
    (64, 8, 128, "bf16", "e4m3", [600, 1, 17, 1024]),
    (32, 8, 128, "f16", "e4m3", [300, 16, 33]),
    (32, 8, 128, "bf16", "int8", [129, 700]),
    (8, 8, 128, "bf16", "e5m2", [100, 1100]),
    (16, 2, 64, "f16", "e4m3", [3, 90, 16]),       # d = 64: CUDA-core kernel
]


@pytest.mark.parametrize("mode,P", [("single", 512), ("split", 512), ("split", 64)])
@pytest.mark.parametrize("case", range(len(PER_CHANNEL)))
def test_per_channel_scales_parity(case, mode, P, kernel_choice):
    """8-bit caches with one scale per (KV head, channel): pools bit-exact
    (pa_cache_write_per_channel) and decode within tolerance."""
    pa, PagedDecode = _pa()
    Hq, Hk, d, act, kv, lens = PER_CHANNEL[case]
    w = workload.build(f"chan{case}", 3000 + case, lens, Hq, Hk, d, act, kv, channel_scales=True,
                       extra_table_cols=1)
    dec = PagedDecode(w, mode=mode, partition_size=P)
    dec.step()
    torch.cuda.synchronize()
    assert dec.error() == 0
    kc, vc = oracle.caches_for(w)
    check_pools(dec, kc, vc)
    assert_close(_to_f64(dec.out), oracle.decode_for(w, kc, vc),
                 f"per-channel case {case} {mode} P={P} kernel={kernel_choice}")


BLOCK32 = [
    # (Hq, Hk, d, act, kv, lens): 32-token pool blocks
    (32, 8, 128, "bf16", "bf16", [1, 31, 32, 33, 100, 513, 700]),
    (4, 2, 64, "f16", "f16", [10, 45, 20, 33]),
    (64, 8, 128, "bf16", "e4m3", [600, 17, 1024]),
    (8, 8, 128, "f16", "int8", [95, 1]),
]


@pytest.mark.parametrize("mode,P", [("single", 512), ("split", 512), ("split", 16), ("fused", 64),
                                    ("fused_single", 512)])
@pytest.mark.parametrize("case", range(len(BLOCK32)))
def test_block_size_32_parity(case, mode, P, kernel_choice):
    """Pools of 32-token blocks (the fifth page's §2.2: blocks of 16-32
    tokens): slot mapping, cache write and append bit-exact, decode within
    tolerance, including 16-token partitions that end inside a block."""
    pa, PagedDecode = _pa()
    Hq, Hk, d, act, kv, lens = BLOCK32[case]
    w = workload.build(f"b32_{case}", 4000 + case, lens, Hq, Hk, d, act, kv, block_size=32,
                       extra_table_cols=1)
    dec = PagedDecode(w, mode=mode, partition_size=P)
    dec.step()
    torch.cuda.synchronize()
    assert dec.error() == 0
    kc, vc = oracle.caches_for(w)
    check_pools(dec, kc, vc)
    assert_close(_to_f64(dec.out), oracle.decode_for(w, kc, vc),
                 f"block 32 case {case} {mode} P={P} kernel={kernel_choice}")


CASCADE = [
    # (Hq, Hk, d, act, lens, shared prefix tokens, block size)
    (8, 8, 128, "f16", [1040, 1030, 1100], 1024, 16),
    (32, 8, 128, "bf16", [100, 65, 66, 700], 64, 16),
    (16, 2, 64, "f16", [33, 40, 300], 32, 16),
    (4, 4, 128, "bf16", [17, 18, 200], 16, 16),
    (32, 8, 128, "f16", [97, 300, 65], 64, 32),
    (24, 8, 64, "bf16", [130, 129], 128, 16),       # GQA 3
    (32, 8, 128, "bf16", [100, 65, 66, 700], 64, 16, "e4m3"),
    (8, 8, 128, "f16", [1040, 1100], 1024, 16, "int8"),
    (16, 4, 128, "bf16", [401, 420, 999], 400, 16),   # 2 prefix key ranges, partial last tile
    (8, 8, 128, "f16", [1041, 1300], 1040, 16),       # 5 ranges, the last one a 16-key tile
]


@pytest.mark.parametrize("P", [16, 512])
@pytest.mark.parametrize("case", range(len(CASCADE)))
def test_shared_prefix_decode_parity(case, P, kernel_choice):
    """pa_decode_shared_prefix: the prefix attended once for all sequences
    (tensor-core pass), tails split, merged -- against the oracle's decode."""
    pa, PagedDecode = _pa()
    Hq, Hk, d, act, lens, prefix, B = CASCADE[case][:7]
    kv = CASCADE[case][7] if len(CASCADE[case]) > 7 else act
    w = workload.build(f"casc{case}", 5000 + case, lens, Hq, Hk, d, act, kv,
                       shared_prefix_tokens=prefix, block_size=B, extra_table_cols=1)
    dec = PagedDecode(w, mode="cascade", partition_size=P)
    out_buf, dec.out = guarded_like(dec.out)
    ws_buf, dec.workspace = guarded_like(dec.workspace)
    dec.step()
    torch.cuda.synchronize()
    assert dec.error() == 0
    check_guards(out_buf, "out")
    check_guards(ws_buf, "workspace")
    kc, vc = oracle.caches_for(w)
    check_pools(dec, kc, vc)
    assert_close(_to_f64(dec.out), oracle.decode_for(w, kc, vc),
                 f"shared prefix case {case} P={P} kernel={kernel_choice}")


def test_shared_prefix_decode_full_size():
    """The continuous-batching workload (256 sequences sharing a 1024-token
    prefix): 64 sampled rows against the oracle, every output inside the
    range of its V rows."""
    pa, PagedDecode = _pa()
    w, kc, vc = _full(5)
    dec = PagedDecode(w, mode="cascade", partition_size=512)
    dec.step()
    torch.cuda.synchronize()
    assert dec.error() == 0
    check_pools(dec, kc, vc)
    out = _to_f64(dec.out)
    pairs = sample_pairs(w, 64, seed=55)
    ref = oracle.decode_for(w, kc, vc, pairs)
    assert_close(out[pairs[:, 0], pairs[:, 1]], ref, "config 5 shared prefix")
    _check_convex_hull(w, dec, out)


def test_shared_prefix_shorter_sequence_is_reported():
    pa, PagedDecode = _pa()
    w = workload.build("cshort", 5100, [80, 90], 8, 2, 64, "f16", "f16", shared_prefix_tokens=64)
    dec = PagedDecode(w, mode="cascade", partition_size=64)
    dec.step()
    torch.cuda.synchronize()
    assert dec.error() == 0
    dec.seq_lens[1] = 40  # shorter than the prefix
    dec.attend()
    torch.cuda.synchronize()
    assert dec.error() == pa.PA_ERR_DEVICE_BOUNDS
    assert torch.isfinite(dec.out.float()).all()


@pytest.mark.parametrize("P,chain", [(128, None), (32, "1"), (32, "3")])
def test_split_partials_match_oracle(kernel_choice, P, chain, monkeypatch):
    """Every partition's (lse, o) against the oracle's; with 32-token
    partitions (35 of them) the tensor-core kernel's warps take 1 or 3
    partitions in a row."""
    if chain:
        monkeypatch.setenv("PA369_DECODE_CHAIN", chain)
    pa, PagedDecode = _pa()
    w = workload.build("partials", 77, [1, 16, 17, 100, 513, 1100], 16, 4, 128, "bf16", "bf16")
    dec = PagedDecode(w, mode="split", partition_size=P)
    dec.step()
    torch.cuda.synchronize()
    assert dec.error() == 0
    kc, vc = oracle.caches_for(w)
    NP = -(-int(w.seq_lens.max()) // P)
    pairs = np.array([(s, h) for s in range(w.num_seqs) for h in range(w.num_q_heads)], np.int32)
    lse_ref, o_ref = oracle.split_partials(w.q, w.act_dtype, kc, vc, w.kv_dtype, w.block_tables,
                                           w.seq_lens, w.num_kv_heads, w.softmax_scale, P, NP,
                                           pairs)
    lse, o = pa.split_workspace_views(dec.workspace, w.num_seqs, w.num_q_heads, w.head_dim,
                                      dec.max_seq_len, P)
    lse, o = _to_f64(lse), _to_f64(o)
    for i, (s, h) in enumerate(pairs):
        np_s = -(-int(w.seq_lens[s]) // P)
        assert np.isinf(lse_ref[i, np_s:]).all()
        assert np.allclose(lse[s, h, :np_s], lse_ref[i, :np_s], rtol=1e-5, atol=1e-4)
        assert_close(o[s, h, :np_s], o_ref[i, :np_s], f"partials s={s} h={h}")


def test_single_token_is_exact_v(kernel_choice):
    """L = 1: p = 1 exactly, so the output equals the new token's v bit for bit."""
    pa, PagedDecode = _pa()
    for act in ("f16", "bf16"):
        w = workload.build("l1", 5, [1, 1, 1], 8, 2, 128, act, act)
        for mode in ("single", "split"):
            dec = PagedDecode(w, mode=mode)
            dec.step()
            torch.cuda.synchronize()
            v = dec.v_new.repeat_interleave(w.group, dim=1)
            assert torch.equal(dec.out.view(torch.int16), v.view(torch.int16))


def test_physical_permutation_bitwise(kernel_choice):
    """Moving blocks to other physical ids (tables rewritten) changes nothing."""
    pa, PagedDecode = _pa()
    w = workload.build("perm", 8, [10, 45, 20, 33, 300], 8, 2, 64, "bf16", "bf16", pool_slack=0.5)
    dec = PagedDecode(w, mode="split", partition_size=64)
    dec.step()
    out1 = dec.out.clone()
    perm = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(1)).to(dec.k_cache.device)
    k2, v2 = torch.empty_like(dec.k_cache), torch.empty_like(dec.v_cache)
    k2[perm], v2[perm] = dec.k_cache, dec.v_cache
    dec.k_cache, dec.v_cache = k2, v2
    dec.block_tables = perm.to(torch.int32)[dec.block_tables.long()].contiguous()
    dec.attend()
    torch.cuda.synchronize()
    assert torch.equal(out1.view(torch.int16), dec.out.view(torch.int16))


def test_identical_v_rows_give_that_row():
    pa, PagedDecode = _pa()
    w = workload.build("same_v", 9, [100, 37], 8, 2, 128, "bf16", "bf16")
    w.v_prefill[:] = w.v_prefill[0:1, :, :]
    w.v_new[:] = w.v_prefill[0:1, :, :]
    dec = PagedDecode(w, mode="split", partition_size=32)
    dec.step()
    torch.cuda.synchronize()
    v = dec.v_new[0:1].repeat_interleave(w.group, dim=1).float()
    got = dec.out.float()
    assert (got - v).abs().max().item() <= 2 ** -8 * v.abs().max().item()


# ---------------------------------------------------------------------------
# the five named workloads at full size
# ---------------------------------------------------------------------------

_FULL = {}


def _full(cfg, kv=None):
    key = (cfg, kv)
    if key not in _FULL:
        _FULL.clear()
        chan = kv is not None and kv.endswith("-channel")
        w = workload.config(cfg, kv_dtype=kv.split("-")[0] if kv else None, channel_scales=chan)
        kc, vc = oracle.caches_for(w)
        _FULL[key] = (w, kc, vc)
    return _FULL[key]


@pytest.mark.parametrize("cfg,kv", [(1, None), (2, None), (3, None), (4, None), (5, None),
                                    (4, "e5m2"), (4, "int8"), (4, "e4m3-channel")])
def test_named_workload_parity(cfg, kv):
    """Each named workload at full size, first in exactly the launch
    configuration bench.py times (the workload's default fused step and
    split-KV partition), then split, single-pass and CUDA-core launches on the
    same state, and split-KV at 512-token partitions where the default
    differs."""
    pa, PagedDecode = _pa()
    from paged_kv_cache_369_b200.runner import default_mode, default_partition_size

    w, kc, vc = _full(cfg, kv)
    chan = w.k_chan is not None
    P = default_partition_size(w, cfg)
    mode = "split" if chan else default_mode(cfg)
    dec = PagedDecode(w, mode=mode, partition_size=P)
    dec.step()  # pa_decode_append: the attention launch stores the new tokens
    torch.cuda.synchronize()
    assert dec.error() == 0
    check_pools(dec, kc, vc)
    out_split = _to_f64(dec.out)
    assert np.isfinite(out_split).all()
    pairs = sample_pairs(w, 64 if cfg > 1 else w.num_seqs * w.num_q_heads, seed=cfg)
    ref = oracle.decode_for(w, kc, vc, pairs)
    assert_close(out_split[pairs[:, 0], pairs[:, 1]], ref, f"config {cfg} {mode} P={P}")
    # unfused split attention on the same state
    dec.mode = "split"
    dec.attend()
    torch.cuda.synchronize()
    assert_close(_to_f64(dec.out)[pairs[:, 0], pairs[:, 1]], ref, f"config {cfg} split P={P}")
    if P != 512:  # the other partition size the kernels are tuned for
        dec.partition_size = 512
        need = pa.pa_split_workspace_bytes(w.num_seqs, w.num_q_heads, w.head_dim,
                                           dec.max_seq_len, 512)
        dec.workspace = torch.empty(max(need, 256), dtype=torch.uint8, device="cuda")
        dec.attend()
        torch.cuda.synchronize()
        assert_close(_to_f64(dec.out)[pairs[:, 0], pairs[:, 1]], ref, f"config {cfg} split P=512")
    # single-pass launch on the same state
    dec.mode = "single"
    dec.attend()
    torch.cuda.synchronize()
    assert dec.error() == 0
    out_single = _to_f64(dec.out)
    assert_close(out_single[pairs[:, 0], pairs[:, 1]], ref, f"config {cfg} single")
    # the CUDA-core kernel on the same state
    os.environ["PA369_DECODE_KERNEL"] = "simt"
    try:
        dec.mode = "split"
        dec.attend()
        torch.cuda.synchronize()
    finally:
        del os.environ["PA369_DECODE_KERNEL"]
    assert dec.error() == 0
    assert_close(_to_f64(dec.out)[pairs[:, 0], pairs[:, 1]], ref, f"config {cfg} simt split")
    # property at full size: every output row is a convex combination of its
    # V rows, so it lies inside their per-element range
    _check_convex_hull(w, dec, out_split)


def _check_convex_hull(w, dec, out):
    g = w.group
    vpool = dec.v_cache
    for s in range(w.num_seqs):
        L = int(w.seq_lens[s])
        if L == 0:
            continue
        nb = -(-L // 16)
        ids = dec.block_tables[s, :nb].long()
        rows = vpool[ids]  # [nb, Hk, 16, d]
        if w.kv_dtype == "e4m3":
            rows = rows.view(torch.float8_e4m3fn).float() * w.v_scale
        elif w.kv_dtype in ("e5m2", "int8"):
            rows = rows.float() * w.v_scale
        if w.v_chan is not None:  # per-channel scales replace the per-tensor one
            codes = vpool[ids]
            codes = codes.view(torch.float8_e4m3fn) if w.kv_dtype == "e4m3" else codes
            rows = codes.float() * torch.from_numpy(w.v_chan).to(codes.device)[None, :, None, :]
        else:
            rows = rows.float()
        rows = rows.permute(1, 0, 2, 3).reshape(w.num_kv_heads, nb * 16, w.head_dim)[:, :L]
        lo = rows.min(dim=1).values.repeat_interleave(g, dim=0).cpu().numpy()
        hi = rows.max(dim=1).values.repeat_interleave(g, dim=0).cpu().numpy()
        slack = 1e-2
        assert (out[s] >= lo - slack).all() and (out[s] <= hi + slack).all(), f"seq {s}"


# ---------------------------------------------------------------------------
# device-side range checks: corrupt inputs are reported, never dereferenced
# ---------------------------------------------------------------------------

def test_corrupt_block_table_is_reported(kernel_choice):
    pa, PagedDecode = _pa()
    w = workload.build("bad", 12, [40, 70], 8, 2, 64, "bf16", "bf16")
    for mode in ("single", "split"):
        dec = PagedDecode(w, mode=mode, partition_size=32)
        dec.block_tables[0, 1] = w.num_blocks + 5
        dec.block_tables[1, 2] = -3
        dec.dev_err.zero_()
        dec.attend()
        torch.cuda.synchronize()
        assert dec.error() == pa.PA_ERR_DEVICE_BOUNDS
        assert torch.isfinite(dec.out.float()).all()


def test_bad_lengths_and_slots_are_reported():
    pa, PagedDecode = _pa()
    w = workload.build("badlen", 13, [40, 70], 8, 2, 64, "f16", "f16")
    dec = PagedDecode(w, mode="single")
    dec.seq_lens[1] = dec.block_tables.shape[1] * 16 + 1
    dec.dev_err.zero_()
    dec.attend()
    torch.cuda.synchronize()
    assert dec.error() == pa.PA_ERR_DEVICE_BOUNDS
    assert torch.isfinite(dec.out.float()).all()
    # slot mapping: sequence index out of range -> slot -1 + error
    dec.dev_err.zero_()
    tseq = torch.tensor([0, 7, -1], dtype=torch.int32, device="cuda")
    tpos = torch.tensor([3, 0, 0], dtype=torch.int32, device="cuda")
    slots = torch.empty(3, dtype=torch.int64, device="cuda")
    pa.pa_slot_mapping(slots, dec.block_tables, dec.seq_lens, tseq, tpos, 3, 2, w.num_blocks,
                       16, dec.dev_err)
    torch.cuda.synchronize()
    assert dec.error() == pa.PA_ERR_DEVICE_BOUNDS
    assert slots.tolist()[1:] == [-1, -1]
    assert slots.tolist()[0] == int(w.block_tables[0, 0]) * 16 + 3
    # cache write: slot past the pool is skipped and reported
    dec.dev_err.zero_()
    before = dec.k_cache.clone()
    bad = torch.tensor([w.num_blocks * 16 + 3, -1], dtype=torch.int64, device="cuda")
    pa.pa_cache_write(dec.k_new, dec.v_new, dec.k_cache, dec.v_cache, bad, dev_err=dec.dev_err)
    torch.cuda.synchronize()
    assert dec.error() == pa.PA_ERR_DEVICE_BOUNDS
    assert torch.equal(before.view(torch.int16), dec.k_cache.view(torch.int16))


def test_split_longer_than_max_seq_len_is_reported():
    pa, PagedDecode = _pa()
    w = workload.build("cap", 14, [100, 300], 4, 2, 64, "bf16", "bf16")
    dec = PagedDecode(w, mode="split", partition_size=64)
    dec.max_seq_len = 128  # understates seq 1
    need = pa.pa_split_workspace_bytes(w.num_seqs, w.num_q_heads, w.head_dim, 128, 64)
    dec.workspace = torch.empty(need, dtype=torch.uint8, device="cuda")
    dec.dev_err.zero_()
    dec.attend()
    torch.cuda.synchronize()
    assert dec.error() == pa.PA_ERR_DEVICE_BOUNDS
    assert torch.isfinite(dec.out.float()).all()
