"""GPU parity of the copy-on-write block copy (pa_copy_blocks) against the
CPU oracle, alone and inside a beam-search fork followed by a decode step.

Bars: pools bit-exact (poison bytes included); attention within max-abs 1e-2
and relative L2 2e-3 of the fp64 oracle."""

import numpy as np
import pytest
import torch

import oracle
import workload
from tests.test_gpu_parity import assert_close, pool_bytes, sample_pairs

pytestmark = pytest.mark.gpu

_TORCH = {"f16": torch.float16, "bf16": torch.bfloat16, "e4m3": torch.uint8}


def _pa():
    import paged_kv_cache_369_b200 as pa
    from paged_kv_cache_369_b200.runner import PagedDecode

    return pa, PagedDecode


def _to_dev(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype != "e4m3":
        t = t.view(torch.int16).view(_TORCH[dtype])
    return t.cuda()


@pytest.mark.parametrize("kv,Hk,d,B", [("f16", 2, 64, 16), ("bf16", 8, 128, 16), ("e4m3", 8, 128, 16),
                                       ("bf16", 1, 64, 16), ("e4m3", 32, 128, 16),
                                       ("bf16", 8, 128, 32)])
def test_copy_blocks_bitwise(kv, Hk, d, B):
    pa, _ = _pa()
    rng = np.random.default_rng({"f16": 1, "bf16": 2, "e4m3": 3}[kv] * 1000 + Hk * 10 + d + B)
    nb = 96
    dt = np.uint8 if kv == "e4m3" else np.uint16
    kc = rng.integers(0, np.iinfo(dt).max, size=(nb, Hk, B, d), dtype=dt)
    vc = rng.integers(0, np.iinfo(dt).max, size=(nb, Hk, B, d), dtype=dt)
    ids = rng.permutation(nb)
    pairs = np.stack([ids[:40], ids[40:80]], 1).astype(np.int32)
    pairs = np.concatenate([pairs, [[int(ids[90]), int(ids[90])]]]).astype(np.int32)  # src == dst
    gk, gv = _to_dev(kc, kv), _to_dev(vc, kv)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_copy_blocks(gk, gv, torch.from_numpy(pairs).cuda(), err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert oracle.copy_blocks(kc, vc, pairs) == 0
    assert np.array_equal(pool_bytes(gk), kc.view(np.uint8).reshape(pool_bytes(gk).shape))
    assert np.array_equal(pool_bytes(gv), vc.view(np.uint8).reshape(pool_bytes(gv).shape))


def test_copy_blocks_out_of_range_is_reported():
    pa, _ = _pa()
    nb = 8
    gk = torch.full((nb, 2, 16, 64), 3.0, dtype=torch.float16, device="cuda")
    gv = torch.full((nb, 2, 16, 64), 5.0, dtype=torch.float16, device="cuda")
    gk[1] = 7.0
    before = gk.clone(), gv.clone()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pairs = torch.tensor([[1, 8], [-1, 2], [1, 2]], dtype=torch.int32, device="cuda")
    pa.pa_copy_blocks(gk, gv, pairs, err)
    torch.cuda.synchronize()
    assert int(err.item()) == pa.PA_ERR_DEVICE_BOUNDS
    want = before[0].clone()
    want[2] = before[0][1]
    assert torch.equal(gk, want) and torch.equal(gv, before[1])


def _fork(w, rng):
    """Beam-search fork of every sequence just before its new token: candidate
    A keeps the table; candidate B gets a fresh block for the logical block
    the new token goes to, a copy of the shared one when that block already
    holds earlier tokens (copy-on-write).  Returns the 2S-sequence batch
    (tables, lens, q, k_new, v_new as raw bits) and the copy pairs."""
    S = w.num_seqs
    free = [int(b) for b in w.free_blocks[1:]]  # free_blocks[0] backs the unused table columns
    tb = w.block_tables.copy()
    pairs = []
    for s in range(S):
        L = int(w.seq_lens[s])
        lb = (L - 1) // w.block_size
        fresh = free.pop(0)
        if (L - 1) % w.block_size:
            pairs.append((int(w.block_tables[s, lb]), fresh))
        tb[s, lb] = fresh
    tables = np.concatenate([w.block_tables, tb]).astype(np.int32)
    lens = np.concatenate([w.seq_lens, w.seq_lens]).astype(np.int32)
    draw = lambda shape: workload.draw_normal_bits(rng, shape, w.act_dtype)
    q = np.concatenate([w.q, draw(w.q.shape)])
    kn = np.concatenate([w.k_new, draw(w.k_new.shape)])
    vn = np.concatenate([w.v_new, draw(w.v_new.shape)])
    return tables, lens, q, kn, vn, np.array(pairs, np.int32).reshape(-1, 2)


def _fork_and_decode(w, seed):
    """GPU: prefill, pa_copy_blocks, then one pa_decode_append over both
    candidates.  Oracle: the same steps on its own pools."""
    pa, PagedDecode = _pa()
    rng = np.random.default_rng(seed)
    tables, lens, q, kn, vn, pairs = _fork(w, rng)
    dec = PagedDecode(w, mode="single")  # pools holding the tokens before this step
    dev = dec.k_cache.device
    t_pairs = torch.from_numpy(pairs).to(dev)
    pa.pa_copy_blocks(dec.k_cache, dec.v_cache, t_pairs, dec.dev_err)
    tq, tkn, tvn = (_to_dev(a, w.act_dtype) for a in (q, kn, vn))
    ttab, tlen = torch.from_numpy(tables).to(dev), torch.from_numpy(lens).to(dev)
    out = torch.empty_like(tq)
    pa.pa_decode_append(out, tq, tkn, tvn, dec.k_cache, dec.v_cache, ttab, tlen, w.softmax_scale,
                        0, int(lens.max()), None, w.k_scale, w.v_scale, dec.dev_err)
    torch.cuda.synchronize()
    assert dec.error() == 0

    kc, vc = oracle.caches_for(w, include_new=False)
    assert oracle.copy_blocks(kc, vc, pairs) == 0
    S2 = 2 * w.num_seqs
    slots = oracle.slot_mapping(tables, lens, np.arange(S2, dtype=np.int32), None, S2,
                                w.block_size)
    oracle.cache_write(kn, vn, kc, vc, slots, w.num_blocks, w.num_kv_heads, w.head_dim,
                       w.block_size, w.act_dtype, w.kv_dtype, w.k_scale, w.v_scale)
    assert np.array_equal(pool_bytes(dec.k_cache), kc.view(np.uint8).reshape(pool_bytes(dec.k_cache).shape))
    assert np.array_equal(pool_bytes(dec.v_cache), vc.view(np.uint8).reshape(pool_bytes(dec.v_cache).shape))
    return out, q, kc, vc, tables, lens


@pytest.mark.parametrize("case", [
    # (lens, Hq, Hk, d, act, kv)
    ([10, 45, 20, 33], 4, 2, 64, "f16", "f16"),
    ([17, 1, 64, 100, 513], 32, 8, 128, "bf16", "bf16"),
    ([600, 2, 18, 1025], 64, 8, 128, "bf16", "e4m3"),
])
def test_fork_copy_then_decode(case):
    lens, Hq, Hk, d, act, kv = case
    nblk = sum(-(-L // 16) for L in lens)
    w = workload.build("fork", 4242 + Hq, lens, Hq, Hk, d, act, kv,
                       num_blocks=nblk + len(lens) + 4, extra_table_cols=1)
    out, q, kc, vc, tables, lens2 = _fork_and_decode(w, 5)
    ref = oracle.decode(q, w.act_dtype, kc, vc, w.kv_dtype, tables, lens2, w.num_kv_heads,
                        w.softmax_scale, w.k_scale, w.v_scale, w.block_size)
    got = out.float().cpu().numpy().astype(np.float64)
    assert_close(got, ref, f"fork {case}")
    # the two candidates differ only through their new token
    S = len(lens)
    assert not np.array_equal(got[:S], got[S:])


def test_fork_copy_then_decode_qwen3_8b_shape():
    """Every sequence of the Qwen3-8B-shaped workload forks (64 copies of
    32 KiB blocks per pool); pools bit-exact, 64 sampled rows vs the oracle."""
    w = workload.config(2)
    out, q, kc, vc, tables, lens2 = _fork_and_decode(w, 6)

    class _W:  # the forked batch, for sample_pairs
        num_seqs, num_q_heads, seq_lens = 2 * w.num_seqs, w.num_q_heads, lens2

    pairs = sample_pairs(_W, 64, seed=3)
    ref = oracle.decode(q, w.act_dtype, kc, vc, w.kv_dtype, tables, lens2, w.num_kv_heads,
                        w.softmax_scale, w.k_scale, w.v_scale, w.block_size, pairs)
    got = out.float().cpu().numpy().astype(np.float64)[pairs[:, 0], pairs[:, 1]]
    assert_close(got, ref, "fork config 2 sampled rows")
