"""The seeded generator: determinism and the structure of the five workloads."""

import numpy as np
import pytest

import workload


def test_deterministic():
    a, b = workload.config(1), workload.config(1)
    for f in ("seq_lens", "block_tables", "q", "k_new", "v_new", "k_prefill", "v_prefill"):
        assert np.array_equal(getattr(a, f), getattr(b, f))


@pytest.mark.parametrize("cfg", [1, 2, 3, 5])
def test_config_structure(cfg):
    w = workload.config(cfg, draw_kv=False)
    S = w.num_seqs
    assert w.block_tables.shape[0] == S
    nblk = -(-w.seq_lens // 16)
    used = set()
    for s in range(S):
        row = w.block_tables[s, :nblk[s]]
        assert ((row >= 0) & (row < w.num_blocks)).all()
        if cfg == 5:
            assert np.array_equal(row[:64], w.block_tables[0, :64])
            used.update(row[64:].tolist())
        else:
            assert not used.intersection(row.tolist())
            used.update(row.tolist())
        # unused columns point at a free (poisoned) block
        assert set(w.block_tables[s, nblk[s]:].tolist()) <= set(w.free_blocks.tolist())
    free = set(w.free_blocks.tolist())
    assert not free.intersection(used)
    if cfg == 1:
        assert w.seq_lens.tolist() == [10, 45, 20, 33] and w.num_blocks == 32
        assert (w.num_q_heads, w.num_kv_heads, w.head_dim, w.act_dtype) == (4, 2, 64, "f16")
    if cfg == 2:
        assert S == 64 and w.seq_lens.min() >= 512 and w.seq_lens.max() <= 4096
        assert (w.num_q_heads, w.num_kv_heads, w.head_dim, w.act_dtype) == (32, 8, 128, "bf16")
    if cfg == 3:
        assert S == 32 and w.seq_lens.min() >= 2048 and w.seq_lens.max() <= 2560
        assert (w.num_q_heads, w.num_kv_heads) == (64, 8)
    if cfg in (2, 3):
        assert w.num_blocks == int(np.ceil(nblk.sum() * 1.1))
    if cfg == 5:
        assert S == 256 and (w.num_q_heads, w.num_kv_heads, w.act_dtype) == (32, 32, "f16")
        tails = w.seq_lens - 1024
        assert tails.min() >= 1 and tails.max() <= 2048
        assert 200 < tails.mean() < 400  # lognormal, pre-clip mean 300
        assert (w.refcount[w.block_tables[0, :64]] == 256).all()


def test_config4_shape_only():
    w = workload.config(4, draw_kv=False)
    assert w.num_seqs == 8 and (w.seq_lens == 32768).all()
    assert w.kv_dtype == "e4m3" and w.act_dtype == "bf16"
    assert w.kv_bytes_logical() == 536870912


def test_prefill_covers_all_but_new_token():
    w = workload.config(5)
    seen = {}
    for s, p in zip(w.prefill_seq, w.prefill_pos):
        seen.setdefault(int(s), set()).add(int(p))
    assert seen[0] >= set(range(1024))
    for s in range(1, w.num_seqs):
        assert seen.get(s, set()) == set(range(1024, int(w.seq_lens[s]) - 1))


def test_e4m3_scale_is_amax_over_448():
    w = workload.build("s", 3, [20, 30], 4, 2, 32, "bf16", "e4m3")
    k = np.concatenate([workload.bits_to_f32(w.k_prefill, "bf16").ravel(),
                        workload.bits_to_f32(w.k_new, "bf16").ravel()])
    assert w.k_scale == float(np.float32(np.abs(k).max()) / np.float32(448))


@pytest.mark.parametrize("kv", ["e4m3", "e5m2", "int8"])
def test_chunked_8bit_scale_is_amax_over_largest_code(kv):
    """Chunked workloads with an 8-bit cache: per-tensor scales over every
    context and chunk row, as for decode."""
    w = workload.build_chunked("c8", 4, [10, 0], [7, 12], 4, 2, 32, "f16", kv)
    for rows, scale in (((w.k_ctx, w.k_chunk), w.k_scale), ((w.v_ctx, w.v_chunk), w.v_scale)):
        x = np.concatenate([workload.bits_to_f32(r, "f16").ravel() for r in rows])
        largest = {"e4m3": 448.0, "e5m2": 57344.0, "int8": 127.0}[kv]  # each format's largest code
        assert scale == float(np.float32(np.abs(x).max()) / np.float32(largest))


def test_chunked_structure():
    """A chunk is the last n of a sequence's L tokens; the context is the rest."""
    w = workload.build_chunked("cs", 9, [5, 0, 33], [4, 9, 1], 8, 2, 64, "bf16", "bf16")
    assert w.query_start.tolist() == [0, 4, 13, 14]
    assert w.seq_lens.tolist() == [9, 9, 34]
    for s in range(w.num_seqs):
        L, n = int(w.seq_lens[s]), int(w.query_start[s + 1] - w.query_start[s])
        assert sorted(w.chunk_pos[w.chunk_seq == s].tolist()) == list(range(L - n, L))
        assert sorted(w.ctx_pos[w.ctx_seq == s].tolist()) == list(range(0, L - n))


def test_prefill_config_with_8bit_cache():
    """--op prefill --kv: the same sequences and shapes with an 8-bit cache."""
    a, b = workload.prefill_config(1), workload.prefill_config(1, kv_dtype="int8")
    assert b.kv_dtype == "int8" and a.kv_dtype == "bf16"
    assert np.array_equal(a.seq_lens, b.seq_lens) and np.array_equal(a.query_start, b.query_start)
    assert (b.num_q_heads, b.num_kv_heads, b.head_dim) == (a.num_q_heads, a.num_kv_heads, a.head_dim)
    assert b.k_scale > 0 and b.v_scale > 0 and "int8" in b.name
