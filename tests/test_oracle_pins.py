"""Pins for the CPU oracle: facts the pages print, library routines, closed
forms, invariants and brute force.  None of these re-types the oracle's own
formulas; each would fail on a plausible slip in it (a wrong index, a dropped
term, a swapped operand, a wrong exponent bias)."""

import json
import math
import os

import numpy as np
import pytest
import torch

import workload

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# block table worked example ("Transformer 推理优化", §3.3)
# ---------------------------------------------------------------------------

def test_block_table_worked_example_layout(orc, golden_dir):
    ex = _load(golden_dir, "block_table_example.json")
    B = ex["block_size"]
    owner = {}
    for name, seq in ex["sequences"].items():
        assert orc.blocks_for_len(seq["tokens"], B) == seq["blocks"] == len(seq["table"])
        for pos in range(seq["tokens"]):
            sl = orc.slot(seq["table"], pos, B)
            phys, off = divmod(sl, B)
            assert off == pos % B
            owner.setdefault(phys, set()).add(f"{name}_{pos // B}")
    layout = []
    for phys in range(ex["num_physical_blocks"]):
        tags = owner.get(phys, set())
        assert len(tags) <= 1
        layout.append(tags.pop() if tags else "free")
    assert layout == ex["physical_layout"]
    assert [p for p in range(ex["num_physical_blocks"]) if p not in owner] == ex["free_blocks"]


def test_block_table_worked_example_spot_slots(orc, golden_dir):
    ex = _load(golden_dir, "block_table_example.json")
    A, Bq = ex["sequences"]["A"]["table"], ex["sequences"]["B"]["table"]
    # A's last token (44) is in logical block 2 -> physical 0, offset 12
    assert orc.slot(A, 44) == 0 * 16 + 12
    # A token 16 opens logical block 1 -> physical 5
    assert orc.slot(A, 16) == 5 * 16
    # B's last token (19) -> logical block 1 -> physical 3, offset 3
    assert orc.slot(Bq, 19) == 3 * 16 + 3


def test_block_table_worked_example_cache_write(orc, golden_dir):
    """Write distinct rows for every token of A and B through the oracle's
    slot mapping and cache write; each physical block must then hold exactly
    the tokens the printed layout assigns to it, and free blocks stay untouched."""
    ex = _load(golden_dir, "block_table_example.json")
    B, nb, d, Hk = 16, ex["num_physical_blocks"], 4, 1
    seqs = [ex["sequences"]["A"], ex["sequences"]["B"]]
    mbs = 3
    bt = np.zeros((2, mbs), np.int32)
    for s, seq in enumerate(seqs):
        bt[s, :len(seq["table"])] = seq["table"]
    tseq = np.concatenate([np.full(seq["tokens"], s, np.int32) for s, seq in enumerate(seqs)])
    tpos = np.concatenate([np.arange(seq["tokens"], dtype=np.int32) for seq in seqs])
    T = tseq.size
    rows = np.zeros((T, Hk, d), np.uint16)
    rows[:, 0, 0] = tseq + 1
    rows[:, 0, 1] = tpos
    kc = orc.empty_pool(nb, Hk, B, d, "f16")
    vc = orc.empty_pool(nb, Hk, B, d, "f16")
    slots = orc.slot_mapping(bt, None, tseq, tpos, T, B)
    assert orc.cache_write(rows, rows, kc, vc, slots, nb, Hk, d, B, "f16", "f16") == 0
    for phys, tag in enumerate(ex["physical_layout"]):
        blk = kc[phys, 0]
        if tag == "free":
            assert (blk == 0xFFFF).all()
            continue
        name, lb = tag.split("_")
        s = 0 if name == "A" else 1
        ntok = seqs[s]["tokens"]
        for off in range(B):
            pos = int(lb) * B + off
            if pos < ntok:
                assert blk[off, 0] == s + 1 and blk[off, 1] == pos
            else:
                assert (blk[off] == 0xFFFF).all()  # unused tail slot untouched


def test_block_counts_printed(orc, golden_dir):
    g = _load(golden_dir, "block_counts.json")
    for case in g["printed"]:
        n = orc.blocks_for_len(case["tokens"], g["block_size"])
        if "page_error" in case:
            # 1000 tokens: the page prints 64 blocks; 16-token blocks give 63
            assert n == 63 and n * 16 >= case["tokens"] and (n - 1) * 16 < case["tokens"]
        else:
            assert n == case["blocks"]
            if "capacity" in case:
                assert n * g["block_size"] == case["capacity"]


def test_utilisation_waste_below_one_block(orc):
    """Only the last block is partly filled: waste < block_size per sequence
    (first page §3.4); utilisation of the large decode workloads > 96 %."""
    rng = np.random.default_rng(0)
    for L in rng.integers(1, 5000, size=200):
        n = orc.blocks_for_len(int(L), 16)
        assert 0 <= n * 16 - L < 16
    for cfg in (2, 3, 5):
        w = workload.config(cfg, draw_kv=False)
        used_blocks = sum(orc.blocks_for_len(int(L), 16) for L in w.seq_lens)
        if cfg == 5:  # the shared prefix is stored once
            used_blocks -= (w.num_seqs - 1) * w.shared_prefix_blocks
            tokens = 1024 + int((w.seq_lens - 1024).sum())
        else:
            tokens = int(w.seq_lens.sum())
        assert tokens / (16 * used_blocks) > 0.96


# ---------------------------------------------------------------------------
# KV-size formula (first page §2.5; openeuler page §2.2)
# ---------------------------------------------------------------------------

def test_kv_bytes_per_token_formula(orc, golden_dir):
    g = _load(golden_dir, "kv_size.json")
    q3 = g["cases"][0]
    per_tok = orc.kv_bytes_per_token(q3["layers"], q3["kv_heads"], q3["head_dim"], q3["bytes"])
    assert per_tok == q3["bytes_per_token"] == 147456
    unit = {"MiB": 2 ** 20, "GiB": 2 ** 30, "GB": 1e9}
    for n, val, u in q3["per_request"]:
        assert abs(per_tok * n / unit[u] - val) <= 0.05 * val + 1e-9
    for n, val, u in q3["ten_concurrent"]:
        assert abs(10 * per_tok * n / unit[u] - val) <= 0.05 * val + 1e-9
    ll = g["cases"][1]
    per_tok70 = orc.kv_bytes_per_token(ll["layers"], ll["kv_heads"], ll["head_dim"], ll["bytes"])
    assert per_tok70 == 327680
    for n, val, u in ll["per_request"]:
        gb = per_tok70 * n / unit[u]
        assert val <= gb < val + 0.1  # printed to one decimal, truncated
    for n, conc in ll["concurrency_in_10GB"]:
        assert math.floor(10e9 / (per_tok70 * n)) == conc


# ---------------------------------------------------------------------------
# element formats: library routines (numpy float16, torch bfloat16 / e4m3fn)
# ---------------------------------------------------------------------------

def test_f16_decode_exhaustive_vs_numpy(orc):
    codes = np.arange(65536, dtype=np.uint16)
    ref = codes.view(np.float16).astype(np.float64)
    got = np.array([orc.lib().orc_f16_decode(int(c)) for c in codes])
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    m = ~np.isnan(ref)
    assert np.array_equal(ref[m], got[m])


def test_bf16_decode_exhaustive_vs_torch(orc):
    codes = np.arange(65536, dtype=np.uint16)
    ref = torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = np.array([orc.lib().orc_bf16_decode(int(c)) for c in codes])
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    m = ~np.isnan(ref)
    assert np.array_equal(ref[m], got[m])


def _torch_e4m3_decode(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def test_e4m3_decode_all_codes_vs_torch(orc):
    codes = np.arange(256, dtype=np.uint8)
    ref = _torch_e4m3_decode(codes)
    got = np.array([orc.e4m3_decode(int(c)) for c in codes])
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    assert np.isnan(got).sum() == 2  # S.1111.111 only
    m = ~np.isnan(ref)
    assert np.array_equal(ref[m], got[m])


def test_e4m3_range_printed(orc, golden_dir):
    g = _load(golden_dir, "fp8_ranges.json")["e4m3"]
    finite = [orc.e4m3_decode(c) for c in range(256) if not math.isnan(orc.e4m3_decode(c))]
    assert max(finite) == g["max_abs"] and min(finite) == -g["max_abs"]
    assert orc.e4m3_encode(1e30) == 0x7E and orc.e4m3_encode(-1e30) == 0xFE


def test_e4m3_encode_identity_and_midpoints_vs_torch(orc):
    vals = sorted({orc.e4m3_decode(c) for c in range(128) if not math.isnan(orc.e4m3_decode(c))})
    # every representable value encodes to itself (both signs)
    for c in range(256):
        v = orc.e4m3_decode(c)
        if math.isnan(v):
            continue
        assert orc.e4m3_encode(v) == c
    # midpoints between neighbours: exact ties, round half to even
    mids = [(a + b) / 2 for a, b in zip(vals[:-1], vals[1:])]
    mids = np.array(mids + [-m for m in mids], dtype=np.float64)
    assert np.all(mids.astype(np.float32).astype(np.float64) == mids)  # exact in fp32
    ours = np.array([orc.e4m3_encode(m) for m in mids], dtype=np.uint8)
    ref = torch.from_numpy(mids.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)
    for m, c in zip(mids, ours):
        assert (c & 1) == 0 or (c & 0x7F) == 0x7E  # even fraction code


def test_e4m3_encode_random_vs_torch(orc):
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.standard_normal(20000) * 4,
        rng.uniform(-460, 460, 5000),
        rng.standard_normal(5000) * 2.0 ** -8,  # subnormal range
        np.array([0.0, -0.0, 2.0 ** -10, -(2.0 ** -10), 447.9, 448.0, -448.0, 463.9]),
    ]).astype(np.float32)
    ours = np.array([orc.lib().orc_e4m3_encode(float(v)) for v in x], dtype=np.uint8)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_saturation_and_nan(orc):
    # beyond the largest finite value the cache saturates (torch would give NaN)
    for v in (464.0, 480.0, 1000.0, float("inf")):
        assert orc.e4m3_encode(v) == 0x7E
        assert orc.e4m3_encode(-v) == 0xFE
    assert orc.e4m3_encode(float("nan")) == 0x7F


# ---------------------------------------------------------------------------
# attention: torch SDPA (fp64) on contiguous rows, closed forms, invariants
# ---------------------------------------------------------------------------

def _contiguous_kv(w):
    """Place every token's K/V rows by (sequence, position) -- no block table
    involved -- as fp64 [S][L_s, Hk, d] lists."""
    f = lambda bits: workload.bits_to_f32(bits, w.act_dtype).astype(np.float64)
    K = [np.zeros((int(L), w.num_kv_heads, w.head_dim)) for L in w.seq_lens]
    V = [np.zeros((int(L), w.num_kv_heads, w.head_dim)) for L in w.seq_lens]
    kp, vp = f(w.k_prefill), f(w.v_prefill)
    for i, (s, p) in enumerate(zip(w.prefill_seq, w.prefill_pos)):
        if w.shared_prefix_blocks and s == 0 and p < 16 * w.shared_prefix_blocks:
            for s2 in range(w.num_seqs):
                K[s2][p], V[s2][p] = kp[i], vp[i]
        else:
            K[s][p], V[s][p] = kp[i], vp[i]
    kn, vn = f(w.k_new), f(w.v_new)
    for s in range(w.num_seqs):
        K[s][w.seq_lens[s] - 1], V[s][w.seq_lens[s] - 1] = kn[s], vn[s]
    return K, V


def _sdpa_ref(w, K, V):
    q = workload.bits_to_f32(w.q, w.act_dtype).astype(np.float64)
    out = np.zeros((w.num_seqs, w.num_q_heads, w.head_dim))
    for s in range(w.num_seqs):
        qs = torch.from_numpy(q[s])[None, :, None, :]  # [1, Hq, 1, d]
        ks = torch.from_numpy(K[s].transpose(1, 0, 2).copy())[None]  # [1, Hk, L, d]
        vs = torch.from_numpy(V[s].transpose(1, 0, 2).copy())[None]
        o = torch.nn.functional.scaled_dot_product_attention(
            qs, ks, vs, scale=w.softmax_scale, enable_gqa=True)
        out[s] = o[0, :, 0, :].numpy()
    return out


@pytest.mark.parametrize("hq,hk,d,act,lens,prefix", [
    (4, 2, 64, "f16", [10, 45, 20, 33], 0),
    (8, 2, 32, "bf16", [1, 16, 17, 40, 3], 0),
    (6, 3, 16, "f16", [33, 48, 49], 32),
    (4, 4, 8, "bf16", [5, 2, 31], 0),
    (8, 1, 64, "bf16", [70], 0),
])
def test_decode_vs_torch_sdpa(orc, hq, hk, d, act, lens, prefix):
    w = workload.build("pin", 11 + hq + d, lens, hq, hk, d, act, act, shared_prefix_tokens=prefix)
    kc, vc = orc.caches_for(w)
    got = orc.decode_for(w, kc, vc)
    K, V = _contiguous_kv(w)
    ref = _sdpa_ref(w, K, V)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_decode_fp8_vs_torch_sdpa_on_dequantised(orc):
    w = workload.build("pin8", 5, [9, 40, 23], 8, 2, 32, "bf16", "e4m3")
    kc, vc = orc.caches_for(w)
    got = orc.decode_for(w, kc, vc)
    # dequantise the identical codes with torch's e4m3 decoder, per token by slot
    K, V = _contiguous_kv(w)
    for s in range(w.num_seqs):
        for t in range(int(w.seq_lens[s])):
            phys, off = w.block_tables[s, t // 16], t % 16
            K[s][t] = _torch_e4m3_decode(kc[phys, :, off, :]) * w.k_scale
            V[s][t] = _torch_e4m3_decode(vc[phys, :, off, :]) * w.v_scale
    ref = _sdpa_ref(w, K, V)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def _rand_rows(rng, L, d):
    return rng.standard_normal((L, d))


def test_closed_forms(orc):
    rng = np.random.default_rng(3)
    d = 16
    q = rng.standard_normal(d)
    # L = 1: the output is v itself
    K, V = _rand_rows(rng, 1, d), _rand_rows(rng, 1, d)
    o, lse = orc.attention(q, K, V, 0.25)
    assert np.array_equal(o, V[0])
    assert lse == pytest.approx(0.25 * float(q @ K[0]), rel=1e-15)
    # identical V rows: the output is that row
    K = _rand_rows(rng, 37, d)
    V = np.tile(rng.standard_normal(d), (37, 1))
    o, _ = orc.attention(q, K, V, 0.25)
    np.testing.assert_allclose(o, V[0], rtol=1e-14)
    # q = 0: uniform weights, the output is the mean of V; lse = log L
    V = _rand_rows(rng, 37, d)
    o, lse = orc.attention(np.zeros(d), K, V, 0.25)
    np.testing.assert_allclose(o, V.mean(axis=0), rtol=1e-13, atol=1e-15)
    assert lse == pytest.approx(math.log(37), rel=1e-14)
    # one dominant logit: the output is that token's v
    K = _rand_rows(rng, 20, d)
    K[13] = 400.0 * q / np.linalg.norm(q)
    o, _ = orc.attention(q, K, V[:20], 1.0)
    np.testing.assert_allclose(o, V[13], rtol=1e-9, atol=1e-9)
    # two equal logits, the rest far below: the mean of the two rows
    K[5] = K[13]
    o, _ = orc.attention(q, K, V[:20], 1.0)
    np.testing.assert_allclose(o, (V[5] + V[13]) / 2, rtol=1e-9, atol=1e-9)
    # L = 0: zeros and lse = -inf
    o, lse = orc.attention(q, np.zeros((0, d)), np.zeros((0, d)), 1.0)
    assert not o.any() and lse == -math.inf


def test_softmax_scale_and_shift_invariance(orc):
    """Adding a constant to every logit (k_t -> k_t + c q / |q|^2) leaves the
    output unchanged; the logits scale with softmax_scale."""
    rng = np.random.default_rng(4)
    d, L = 32, 50
    q = rng.standard_normal(d)
    K, V = _rand_rows(rng, L, d), _rand_rows(rng, L, d)
    o1, lse1 = orc.attention(q, K, V, 0.3)
    o2, lse2 = orc.attention(q, K + 5.0 * q / (q @ q), V, 0.3)
    np.testing.assert_allclose(o1, o2, rtol=1e-11, atol=1e-13)
    assert lse2 == pytest.approx(lse1 + 0.3 * 5.0, rel=1e-12)
    o3, _ = orc.attention(2 * q, K, V, 0.15)
    np.testing.assert_allclose(o1, o3, rtol=1e-13, atol=1e-14)


def test_physical_permutation_invariance(orc):
    """Relabelling physical blocks (moving blocks and rewriting the tables)
    leaves the output bitwise unchanged."""
    w = workload.build("perm", 21, [10, 45, 20, 33, 64], 8, 2, 32, "bf16", "bf16", pool_slack=0.5)
    kc, vc = orc.caches_for(w)
    base = orc.decode_for(w, kc, vc)
    perm = np.random.default_rng(9).permutation(w.num_blocks)  # old id -> new id
    kc2, vc2 = np.empty_like(kc), np.empty_like(vc)
    kc2[perm], vc2[perm] = kc, vc
    bt2 = perm[w.block_tables].astype(np.int32)
    out2 = orc.decode(w.q, w.act_dtype, kc2, vc2, w.kv_dtype, bt2, w.seq_lens, w.num_kv_heads,
                      w.softmax_scale)
    assert np.array_equal(base, out2)


@pytest.mark.parametrize("B", [1, 8, 32])
def test_block_size_invariance(orc, B):
    """The same logical K/V stored in blocks of 1, 8 or 32 tokens gives the
    bitwise-identical output to 16-token blocks."""
    w = workload.build("bs", 31, [10, 45, 20, 33], 4, 2, 16, "f16", "f16")
    kc, vc = orc.caches_for(w)
    base = orc.decode_for(w, kc, vc)
    K, V = _contiguous_kv(w)
    mbs = max(-(-int(L) // B) for L in w.seq_lens)
    nb = w.num_seqs * mbs
    kcb = orc.empty_pool(nb, w.num_kv_heads, B, w.head_dim, "f16")
    vcb = orc.empty_pool(nb, w.num_kv_heads, B, w.head_dim, "f16")
    bt = np.arange(nb, dtype=np.int32)[::-1].reshape(w.num_seqs, mbs).copy()
    for s in range(w.num_seqs):
        L = int(w.seq_lens[s])
        rows_k = workload.f32_to_bits(K[s].astype(np.float32), "f16")
        rows_v = workload.f32_to_bits(V[s].astype(np.float32), "f16")
        slots = orc.slot_mapping(bt, None, np.full(L, s, np.int32), np.arange(L, dtype=np.int32),
                                 L, B)
        orc.cache_write(rows_k, rows_v, kcb, vcb, slots, nb, w.num_kv_heads, w.head_dim, B,
                        "f16", "f16")
    out = orc.decode(w.q, "f16", kcb, vcb, "f16", bt, w.seq_lens, w.num_kv_heads,
                     w.softmax_scale, block_size=B)
    assert np.array_equal(base, out)


@pytest.mark.parametrize("P", [16, 48, 512])
def test_split_equals_unsplit(orc, P):
    w = workload.build("split", 41, [1, 15, 16, 17, 100, 700], 4, 2, 32, "bf16", "bf16")
    kc, vc = orc.caches_for(w)
    base = orc.decode_for(w, kc, vc)
    NP = -(-int(w.seq_lens.max()) // P)
    pairs = np.array([(s, h) for s in range(w.num_seqs) for h in range(w.num_q_heads)], np.int32)
    lse, o = orc.split_partials(w.q, w.act_dtype, kc, vc, w.kv_dtype, w.block_tables, w.seq_lens,
                                w.num_kv_heads, w.softmax_scale, P, NP, pairs)
    for i, (s, h) in enumerate(pairs):
        merged = orc.split_merge(lse[i], o[i])
        np.testing.assert_allclose(merged, base[s, h], rtol=1e-12, atol=1e-14)
        # partitions past the sequence are empty
        L = int(w.seq_lens[s])
        for p in range(NP):
            if p * P >= L:
                assert lse[i, p] == -math.inf and not o[i, p].any()
        # the partition log-sum-exps combine to the whole-sequence one
        full_lse = orc.split_partials(w.q, w.act_dtype, kc, vc, w.kv_dtype, w.block_tables,
                                      w.seq_lens, w.num_kv_heads, w.softmax_scale, 1 << 20, 1,
                                      pairs[i:i + 1])[0][0, 0]
        finite = lse[i][np.isfinite(lse[i])]
        m = finite.max()
        assert m + math.log(np.exp(finite - m).sum()) == pytest.approx(full_lse, rel=1e-13)


def test_cache_write_then_gather_roundtrip(orc):
    """Brute force: rows written at random slots come back from a gather
    through the same tables; every other byte keeps its poison."""
    rng = np.random.default_rng(5)
    w = workload.build("rt", 51, [3, 16, 17, 40], 4, 2, 64, "bf16", "bf16")
    kc, vc = orc.caches_for(w)
    for s in range(w.num_seqs):
        L = int(w.seq_lens[s])
        K, V = _contiguous_kv(w)
        for h in range(w.num_kv_heads):
            g = orc.gather(kc, "bf16", 1.0, w.block_tables[s], L, w.num_kv_heads, h, w.head_dim)
            np.testing.assert_array_equal(g, K[s][:, h, :])
    # bytes outside the written slots: poison
    written = np.zeros((w.num_blocks, 16), bool)
    for s in range(w.num_seqs):
        for t in range(int(w.seq_lens[s])):
            written[w.block_tables[s, t // 16], t % 16] = True
    assert (kc.transpose(0, 2, 1, 3)[~written] == 0xFFFF).all()
    assert (vc.transpose(0, 2, 1, 3)[~written] == 0xFFFF).all()
    _ = rng


def test_cache_write_fp8_matches_torch_quantiser(orc):
    """E4M3 cache write = torch's e4m3fn cast of (x / scale) computed in fp32,
    for in-range values; negative slots are skipped."""
    rng = np.random.default_rng(6)
    T, Hk, d, nb = 40, 2, 32, 8
    x = rng.standard_normal((T, Hk, d)).astype(np.float32) * 3
    bits = workload.f32_to_bits(x, "bf16")
    xf = workload.bits_to_f32(bits, "bf16")
    scale = np.float32(np.abs(xf).max()) / np.float32(448.0)
    slots = rng.choice(nb * 16, size=T, replace=False).astype(np.int64)
    slots[::7] = -1
    kc = orc.empty_pool(nb, Hk, 16, d, "e4m3")
    vc = orc.empty_pool(nb, Hk, 16, d, "e4m3")
    orc.cache_write(bits, bits, kc, vc, slots, nb, Hk, d, 16, "bf16", "e4m3", float(scale),
                    float(scale))
    ref = torch.from_numpy(xf / scale).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for t in range(T):
        if slots[t] < 0:
            continue
        b, o = divmod(int(slots[t]), 16)
        np.testing.assert_array_equal(kc[b, :, o, :], ref[t])
    touched = {int(s) for s in slots if s >= 0}
    for sl in range(nb * 16):
        if sl not in touched:
            b, o = divmod(sl, 16)
            assert (kc[b, :, o, :] == 0xFF).all()


def test_slot_mapping_decode_form(orc):
    w = workload.config(1)
    slots = orc.slot_mapping(w.block_tables, w.seq_lens, None, None, w.num_seqs)
    for s in range(w.num_seqs):
        pos = int(w.seq_lens[s]) - 1
        assert slots[s] == w.block_tables[s, pos // 16] * 16 + pos % 16
    neg = orc.slot_mapping(w.block_tables, w.seq_lens, np.array([-1, 2], np.int32),
                           np.array([0, 5], np.int32), 2)
    assert neg[0] == -1 and neg[1] == w.block_tables[2, 0] * 16 + 5
