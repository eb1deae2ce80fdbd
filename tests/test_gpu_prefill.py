"""GPU parity of chunked prefill (pa_prefill, tcgen05 tensor cores) against
the CPU oracle.  Bars as for decode: pools bit-exact, attention within
max-abs 1e-2 and relative L2 2e-3 of the fp64 oracle."""

import numpy as np
import pytest
import torch

import oracle
import workload
from tests.test_gpu_parity import assert_close, pool_bytes

pytestmark = pytest.mark.gpu


def _run(w):
    from paged_kv_cache_369_b200.runner import PagedPrefill

    pre = PagedPrefill(w)
    pre.out.view(torch.uint8).fill_(0x7F)  # rows no sequence covers keep this
    pre.step()
    torch.cuda.synchronize()
    return pre


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


SMALL = [
    # (context lens, chunk lens, Hq, Hk, d, dtype)
    ([0, 5, 37, 16], [7, 1, 40, 16], 8, 2, 64, "bf16"),
    ([0, 100, 300], [128, 33, 200], 32, 8, 128, "bf16"),
    ([0, 700], [600, 130], 32, 8, 128, "f16"),
    ([3, 250], [29, 64], 4, 4, 64, "f16"),                  # MHA
    ([0, 64, 1000], [130, 3, 257], 64, 8, 128, "bf16"),     # GQA 8
    ([20, 0, 127], [9, 17, 1], 6, 2, 64, "bf16"),           # GQA 3: 42 tokens per tile
    ([0, 16, 31], [1, 1, 1], 16, 2, 128, "f16"),            # one-token chunks (decode form)
    ([511, 0], [1, 0], 32, 32, 128, "bf16"),                 # an empty chunk
]


@pytest.mark.parametrize("case", range(len(SMALL)))
def test_prefill_small_full_parity(case):
    ctx, chunk, Hq, Hk, d, dt = SMALL[case]
    w = workload.build_chunked(f"pf{case}", 2000 + case, ctx, chunk, Hq, Hk, d, dt, dt,
                               extra_table_cols=2)
    pre = _run(w)
    assert pre.error() == 0
    kc, vc = oracle.chunked_caches_for(w)
    assert np.array_equal(pool_bytes(pre.k_cache), kc.view(np.uint8).reshape(pool_bytes(pre.k_cache).shape))
    assert np.array_equal(pool_bytes(pre.v_cache), vc.view(np.uint8).reshape(pool_bytes(pre.v_cache).shape))
    ref = oracle.prefill_for(w, kc, vc)
    assert_close(_f64(pre.out), ref, f"prefill case {case}")


def _scale_rows(bits, dtype, factor, rows=slice(None)):
    """Multiply the given token rows of 16-bit patterns by a power of two (exact)."""
    f = workload.bits_to_f32(bits, dtype).astype(np.float32)
    f[rows] *= np.float32(factor)
    return workload.f32_to_bits(f, dtype)


@pytest.mark.parametrize("kind", ["huge", "tiny", "early_block", "late_block"])
def test_prefill_bf16_value_range(kind):
    """bf16 caches hold values far outside f16's range, which a P.V in f16
    (V converted per tile with a power-of-two scale) would have to carry and
    the bf16 hi + lo P.V carries as they are: all V times 2^20 or 2^-40, or
    one 16-token block of the context times 2^18, in the first key tile or in
    a later one.  The output must come out as the oracle's.  Each sequence's
    rows are compared after dividing by a power of two near their largest
    magnitude (exact), with the usual bars."""
    w = workload.build_chunked(f"range {kind}", 2900, [0, 230, 90], [150, 40, 64], 32, 8, 128,
                               "bf16", "bf16")
    if kind in ("huge", "tiny"):
        fac = 2.0 ** 20 if kind == "huge" else 2.0 ** -40
        w.v_ctx = _scale_rows(w.v_ctx, "bf16", fac)
        w.v_chunk = _scale_rows(w.v_chunk, "bf16", fac)
    else:
        lo = 16 if kind == "early_block" else 192  # context positions of the scaled block
        rows = np.nonzero((w.ctx_pos >= lo) & (w.ctx_pos < lo + 16))[0]
        w.v_ctx = _scale_rows(w.v_ctx, "bf16", 2.0 ** 18, rows)
    pre = _run(w)
    assert pre.error() == 0
    kc, vc = oracle.chunked_caches_for(w)
    ref = oracle.prefill_for(w, kc, vc)
    got = _f64(pre.out)
    for s in range(w.num_seqs):
        r = slice(int(w.query_start[s]), int(w.query_start[s + 1]))
        if r.start == r.stop:
            continue
        norm = 2.0 ** -np.round(np.log2(np.abs(ref[r]).max()))
        assert_close(got[r] * norm, ref[r] * norm, f"{kind} seq {s}")


def test_prefill_rows_independent_of_chunking_bitwise():
    """One 300-token prompt prefilled as one chunk, or as chunks of 100, 77
    and 123 over the growing cache: every row is bit-identical (each row's
    arithmetic sees only its own keys, in the same key tiles)."""
    from paged_kv_cache_369_b200 import pa_prefill

    full = workload.build_chunked("one", 31, [0], [300], 32, 8, 128, "bf16", "bf16")
    pre = _run(full)
    ref = pre.out.clone()
    start = 0
    for n in (100, 77, 123):
        out = torch.empty((n, 32, 128), dtype=torch.bfloat16, device="cuda")
        lens = torch.tensor([start + n], dtype=torch.int32, device="cuda")
        qs = torch.tensor([0, n], dtype=torch.int32, device="cuda")
        pa_prefill(out, pre.q[start:start + n].contiguous(), pre.k_cache, pre.v_cache,
                   pre.block_tables, lens, qs, n, full.softmax_scale, pre.dev_err)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref[start:start + n].view(torch.int16))
        start += n
    assert pre.error() == 0


def test_prefill_one_token_chunk_matches_decode():
    from paged_kv_cache_369_b200 import pa_decode

    w = workload.build_chunked("dec", 32, [0, 15, 16, 99, 2000], [1] * 5, 32, 8, 128, "bf16", "bf16")
    pre = _run(w)
    out = torch.empty_like(pre.out)
    pa_decode(out, pre.q, pre.k_cache, pre.v_cache, pre.block_tables, pre.seq_lens,
              w.softmax_scale, dev_err=pre.dev_err)
    torch.cuda.synchronize()
    assert pre.error() == 0
    kc, vc = oracle.chunked_caches_for(w)
    ref = oracle.prefill_for(w, kc, vc)
    assert_close(_f64(pre.out), ref, "prefill n=1")
    assert_close(_f64(out), ref, "decode on the same cache")


@pytest.mark.parametrize("cfg", [1, 2])
def test_named_prefill_workload_parity(cfg):
    """The 512-token-chunk workloads at full size: 96 sampled rows (token,
    head) against the oracle, computed on gathered rows; every output finite
    and inside the range of its V rows."""
    w = workload.prefill_config(cfg)
    pre = _run(w)
    assert pre.error() == 0
    got = _f64(pre.out)
    assert np.isfinite(got).all()
    kc, vc = oracle.chunked_caches_for(w)
    rng = np.random.default_rng(cfg)
    S = w.num_seqs
    picks = [(0, 0, 0), (S - 1, w.chunk_lens[-1] - 1, w.num_q_heads - 1)]
    while len(picks) < 96:
        s = int(rng.integers(S))
        picks.append((s, int(rng.integers(w.chunk_lens[s])), int(rng.integers(w.num_q_heads))))
    refs, gots = [], []
    for s, j, h in picks:
        row = int(w.query_start[s]) + j
        L = int(w.seq_lens[s])
        n = int(w.chunk_lens[s])
        kvh = h // w.group
        K = oracle.gather(kc, w.kv_dtype, 1.0, w.block_tables[s], L - n + j + 1, w.num_kv_heads, kvh, w.head_dim)
        V = oracle.gather(vc, w.kv_dtype, 1.0, w.block_tables[s], L - n + j + 1, w.num_kv_heads, kvh, w.head_dim)
        q = workload.bits_to_f32(w.q[row, h], w.act_dtype).astype(np.float64)
        o, _ = oracle.attention(q, K, V, w.softmax_scale)
        refs.append(o)
        gots.append(got[row, h])
        assert (got[row, h] >= V.min(0) - 1e-2).all() and (got[row, h] <= V.max(0) + 1e-2).all()
    assert_close(np.array(gots), np.array(refs), f"prefill config {cfg} sampled rows")


def test_prefill_bad_chunk_is_reported():
    from paged_kv_cache_369_b200 import PA_ERR_DEVICE_BOUNDS, pa_prefill

    w = workload.build_chunked("bad", 33, [10, 20], [5, 6], 8, 2, 64, "f16", "f16")
    pre = _run(w)
    assert pre.error() == 0
    lens = torch.tensor([3, 26], dtype=torch.int32, device="cuda")  # chunk 0 longer than its sequence
    out = torch.zeros_like(pre.out)
    pa_prefill(out, pre.q, pre.k_cache, pre.v_cache, pre.block_tables, lens, pre.query_start,
               w.max_query_len, w.softmax_scale, pre.dev_err)
    torch.cuda.synchronize()
    assert pre.error() == PA_ERR_DEVICE_BOUNDS
    assert not out[:5].any()              # the bad sequence's rows are not written
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("case", [0, 2, 4])
def test_prefill_block_size_32(case):
    """32-token pool blocks: the same small shapes as above."""
    ctx, chunk, Hq, Hk, d, dt = SMALL[case]
    w = workload.build_chunked(f"pf32_{case}", 2100 + case, ctx, chunk, Hq, Hk, d, dt, dt,
                               block_size=32, extra_table_cols=1)
    pre = _run(w)
    assert pre.error() == 0
    kc, vc = oracle.chunked_caches_for(w)
    assert np.array_equal(pool_bytes(pre.k_cache), kc.view(np.uint8).reshape(pool_bytes(pre.k_cache).shape))
    ref = oracle.prefill_for(w, kc, vc)
    assert_close(_f64(pre.out), ref, f"prefill block 32 case {case}")


@pytest.mark.parametrize("case", [
    # (context lens, chunk lens, Hq, Hk, act, kv)
    ([0, 100, 300], [128, 33, 200], 32, 8, "bf16", "e4m3"),
    ([0, 64, 1000], [130, 3, 257], 64, 8, "bf16", "int8"),
    ([3, 250], [29, 64], 4, 4, "f16", "e5m2"),
    ([20, 0, 127], [9, 17, 1], 6, 2, "f16", "e4m3"),
])
def test_prefill_8bit_caches(case):
    """8-bit caches (per-tensor scales): the converter warp widens each tile
    to f16 in shared memory; against the oracle, which dequantises the same
    codes (pools compared bit for bit first)."""
    ctx, chunk, Hq, Hk, act, kv = case
    w = workload.build_chunked(f"pf8_{kv}", 2200 + Hq, ctx, chunk, Hq, Hk, 128, act, kv,
                               extra_table_cols=2)
    pre = _run(w)
    assert pre.error() == 0
    kc, vc = oracle.chunked_caches_for(w)
    assert np.array_equal(pool_bytes(pre.k_cache), kc.view(np.uint8).reshape(pool_bytes(pre.k_cache).shape))
    assert np.array_equal(pool_bytes(pre.v_cache), vc.view(np.uint8).reshape(pool_bytes(pre.v_cache).shape))
    ref = oracle.prefill_for(w, kc, vc)
    assert_close(_f64(pre.out), ref, f"prefill {kv} {case}")
