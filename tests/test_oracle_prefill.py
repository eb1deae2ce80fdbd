"""Pins for the oracle's chunked-prefill attention (openeuler page §4.5;
second page §3.3): torch SDPA in fp64 with an explicit causal mask on
contiguous rows (no block table), the invariance of every query row under
how the prompt is cut into chunks, the decode step as the one-token chunk,
closed forms, and physical-block relabelling."""

import numpy as np
import pytest
import torch

import workload


def _contiguous(w):
    """Per sequence: K, V as fp64 [L, Hk, d] in position order, from the
    generator's rows (context, then chunk) -- no slots, no pools."""
    Ks, Vs = [], []
    for s in range(w.num_seqs):
        L = int(w.seq_lens[s])
        K = np.zeros((L, w.num_kv_heads, w.head_dim))
        V = np.zeros_like(K)
        m = w.ctx_seq == s
        K[w.ctx_pos[m]] = workload.bits_to_f32(w.k_ctx[m], w.act_dtype)
        V[w.ctx_pos[m]] = workload.bits_to_f32(w.v_ctx[m], w.act_dtype)
        m = w.chunk_seq == s
        K[w.chunk_pos[m]] = workload.bits_to_f32(w.k_chunk[m], w.act_dtype)
        V[w.chunk_pos[m]] = workload.bits_to_f32(w.v_chunk[m], w.act_dtype)
        Ks.append(K)
        Vs.append(V)
    return Ks, Vs


def _sdpa_reference(w):
    """torch.nn.functional.scaled_dot_product_attention in fp64, GQA via
    enable_gqa, with the boolean mask key_pos <= query_pos."""
    Ks, Vs = _contiguous(w)
    q = workload.bits_to_f32(w.q, w.act_dtype).astype(np.float64)
    out = np.zeros(q.shape)
    for s in range(w.num_seqs):
        a, b = int(w.query_start[s]), int(w.query_start[s + 1])
        if b == a:
            continue
        L = int(w.seq_lens[s])
        n = b - a
        qpos = np.arange(L - n, L)
        mask = torch.from_numpy(np.arange(L)[None, :] <= qpos[:, None])
        qs = torch.from_numpy(q[a:b]).permute(1, 0, 2)[None]          # [1, Hq, n, d]
        ks = torch.from_numpy(Ks[s]).permute(1, 0, 2)[None]           # [1, Hk, L, d]
        vs = torch.from_numpy(Vs[s]).permute(1, 0, 2)[None]
        o = torch.nn.functional.scaled_dot_product_attention(
            qs, ks, vs, attn_mask=mask, scale=w.softmax_scale, enable_gqa=True)
        out[a:b] = o[0].permute(1, 0, 2).numpy()
    return out


@pytest.mark.parametrize("ctx,chunk,Hq,Hk,d,act", [
    ([0, 5, 37, 16], [7, 1, 40, 16], 8, 2, 32, "bf16"),
    ([3, 100], [29, 64], 4, 4, 64, "f16"),            # MHA
    ([0, 64], [130, 3], 16, 2, 32, "f16"),            # GQA 8
    ([20, 0], [9, 17], 6, 2, 16, "bf16"),             # GQA 3
])
def test_prefill_vs_torch_sdpa_causal(orc, ctx, chunk, Hq, Hk, d, act):
    w = workload.build_chunked("pf", 11 + Hq + d, ctx, chunk, Hq, Hk, d, act, act, pool_slack=0.5)
    kc, vc = orc.chunked_caches_for(w)
    got = orc.prefill_for(w, kc, vc)
    ref = _sdpa_reference(w)
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12)


def _dequantise(codes, kv):
    """8-bit codes to fp64 by torch's fp8 decoders / numpy's int8 view, not the oracle's."""
    if kv == "int8":
        return codes.view(np.int8).astype(np.float64)
    fmt = torch.float8_e4m3fn if kv == "e4m3" else torch.float8_e5m2
    return torch.from_numpy(codes).view(fmt).double().numpy()


@pytest.mark.parametrize("kv", ["e4m3", "e5m2", "int8"])
def test_prefill_8bit_vs_sdpa_on_dequantised(orc, kv):
    w = workload.build_chunked("pf8", 5, [30, 2], [20, 33], 8, 2, 32, "bf16", kv)
    kc, vc = orc.chunked_caches_for(w)
    got = orc.prefill_for(w, kc, vc)
    # rebuild the generator's rows from the codes the oracle stored, decoded independently
    k_deq = _dequantise(kc, kv) * w.k_scale
    v_deq = _dequantise(vc, kv) * w.v_scale
    q = workload.bits_to_f32(w.q, w.act_dtype).astype(np.float64)
    for s in range(w.num_seqs):
        L, a, b = int(w.seq_lens[s]), int(w.query_start[s]), int(w.query_start[s + 1])
        rows = [w.block_tables[s, t // 16] for t in range(L)]
        K = np.stack([k_deq[rows[t], :, t % 16, :] for t in range(L)])
        V = np.stack([v_deq[rows[t], :, t % 16, :] for t in range(L)])
        n = b - a
        mask = torch.from_numpy(np.arange(L)[None, :] <= np.arange(L - n, L)[:, None])
        o = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[a:b]).permute(1, 0, 2)[None],
            torch.from_numpy(K).permute(1, 0, 2)[None], torch.from_numpy(V).permute(1, 0, 2)[None],
            attn_mask=mask, scale=w.softmax_scale, enable_gqa=True)
        np.testing.assert_allclose(got[a:b], o[0].permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)


def test_prefill_rows_do_not_depend_on_chunking(orc):
    """A prompt of 70 tokens prefilled in one chunk, or as chunks of 16, 31
    and 23 tokens over the growing cache: every query row is the same, bit
    for bit (each row attends to exactly the keys at or before it)."""
    full = workload.build_chunked("one", 21, [0], [70], 8, 2, 32, "bf16", "bf16", pool_slack=0.5)
    kc, vc = orc.chunked_caches_for(full)
    ref = orc.prefill_for(full, kc, vc)
    start = 0
    for n in (16, 31, 23):
        qs = np.array([0, n], np.int32)
        lens = np.array([start + n], np.int32)
        got = orc.prefill(full.q[start:start + n], "bf16", kc, vc, "bf16", full.block_tables,
                          lens, qs, full.num_kv_heads, full.softmax_scale)
        assert np.array_equal(got, ref[start:start + n])
        start += n


def test_prefill_one_token_chunk_is_decode(orc):
    w = workload.build_chunked("dec", 22, [0, 15, 16, 99], [1, 1, 1, 1], 8, 2, 64, "f16", "f16")
    kc, vc = orc.chunked_caches_for(w)
    got = orc.prefill_for(w, kc, vc)
    dec = orc.decode(w.q, "f16", kc, vc, "f16", w.block_tables, w.seq_lens, w.num_kv_heads,
                     w.softmax_scale)
    assert np.array_equal(got, dec)


def test_prefill_closed_forms(orc):
    """Position 0 sees only itself: its output is v_0 exactly.  With all
    V rows equal, every output is that row."""
    w = workload.build_chunked("cf", 23, [0, 0], [5, 18], 4, 2, 32, "bf16", "bf16")
    kc, vc = orc.chunked_caches_for(w)
    got = orc.prefill_for(w, kc, vc)
    g = w.group
    for s in range(w.num_seqs):
        row = int(w.query_start[s])
        v0 = workload.bits_to_f32(w.v_chunk[row], "bf16").astype(np.float64)
        for h in range(w.num_q_heads):
            assert np.array_equal(got[row, h], v0[h // g])
    w.v_ctx[:] = w.v_chunk[0]
    w.v_chunk[:] = w.v_chunk[0]
    kc, vc = orc.chunked_caches_for(w)
    got = orc.prefill_for(w, kc, vc)
    v0 = workload.bits_to_f32(w.v_chunk[0], "bf16").astype(np.float64)
    for h in range(w.num_q_heads):
        np.testing.assert_allclose(got[:, h], np.broadcast_to(v0[h // g], got[:, h].shape),
                                   rtol=1e-12, atol=1e-12)


def test_prefill_block_relabelling_bitwise(orc):
    w = workload.build_chunked("perm", 24, [40, 3], [25, 60], 8, 4, 32, "f16", "f16", pool_slack=0.3)
    kc, vc = orc.chunked_caches_for(w)
    ref = orc.prefill_for(w, kc, vc)
    perm = np.random.default_rng(1).permutation(w.num_blocks)
    kc2, vc2 = np.empty_like(kc), np.empty_like(vc)
    kc2[perm], vc2[perm] = kc, vc
    bt2 = perm[w.block_tables].astype(np.int32)
    got = orc.prefill(w.q, "f16", kc2, vc2, "f16", bt2, w.seq_lens, w.query_start,
                      w.num_kv_heads, w.softmax_scale)
    assert np.array_equal(got, ref)


def test_prefill_rejects_chunk_longer_than_sequence(orc):
    w = workload.build_chunked("bad", 25, [0], [4], 2, 2, 16, "f16", "f16")
    kc, vc = orc.chunked_caches_for(w)
    with pytest.raises(ValueError):
        orc.prefill(w.q, "f16", kc, vc, "f16", w.block_tables, np.array([3], np.int32),
                    w.query_start, w.num_kv_heads, w.softmax_scale)


def test_named_prefill_workloads_shapes():
    for cfg in (1, 2):
        w = workload.prefill_config(cfg)
        assert w.max_query_len == 512 and (w.chunk_lens == 512).all()
        assert w.num_tokens == 512 * w.num_seqs
        assert w.flops() > 0
