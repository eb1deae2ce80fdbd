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
