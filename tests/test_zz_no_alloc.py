"""The allocation-free split-KV entry point against the workspace one.

pa_decode_split_reduce_static_scratch serves callers that cannot allocate
device memory (no allocator handed to them, HBM already reserved for the KV
pool, or no room for cudaMalloc's synchronisation on their path): its partials
live in a device array inside the library.  It runs the same partition and
reduce kernels as pa_decode_split_reduce on the same partitions, only with
another scratch address, so its output must equal that entry point's bit for
bit.  This test calls it through the C ABI twice in a row per workload,
checks both outputs for bit equality with pa_decode_split_reduce given a
caller-allocated workspace, and checks the tiny workload against the oracle
within the parity tolerance (max-abs 1e-2, relative L2 2e-3).  One case runs a
large workload and then a small one in the same process: the small call must
not pick up partials the large one left in the shared array.  The file is
collected last and must pass alone in a fresh process as well as after every
other test (the first call in a context does the one-time address lookup)."""

import numpy as np
import pytest
import torch

import oracle
import workload

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
REL_L2 = 2e-3


def _call_static(pa, dec, out, P):
    w = dec.w
    return pa.lib().pa_decode_split_reduce_static_scratch(
        out.data_ptr(), dec.q.data_ptr(), dec.k_cache.data_ptr(), dec.v_cache.data_ptr(),
        dec.block_tables.data_ptr(), int(dec.block_tables.shape[1]), dec.seq_lens.data_ptr(),
        w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, w.num_blocks,
        float(w.softmax_scale), pa.dtype_code(dec.q.dtype), pa.dtype_code(dec.k_cache.dtype),
        float(w.k_scale), float(w.v_scale), P, dec.max_seq_len, dec.dev_err.data_ptr(),
        torch.cuda.current_stream().cuda_stream)


def _decoder(cfg, P):
    """A workload resident on the GPU with its new tokens written and its
    output computed by pa_decode_split_reduce with a torch-allocated workspace."""
    from paged_kv_cache_369_b200.runner import PagedDecode

    dec = PagedDecode(workload.config(cfg), mode="split", partition_size=P)
    dec.step()
    torch.cuda.synchronize()
    assert dec.error() == 0
    return dec, dec.out.clone()


def _static_twice(pa, dec, ref, P):
    out = torch.empty_like(ref)
    for _ in range(2):  # two calls in a row share (and reuse) the library's array
        out.fill_(float("nan"))
        status = _call_static(pa, dec, out, P)
        torch.cuda.synchronize()
        assert status == pa.PA_OK, pa.pa_status_string(status)
        assert dec.error() == 0
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    return out


@pytest.mark.parametrize("cfg", [1, 2, 4])
def test_static_scratch_matches_workspace_entry_point(cfg):
    import paged_kv_cache_369_b200 as pa

    P = 512
    dec, ref = _decoder(cfg, P)
    out = _static_twice(pa, dec, ref, P)
    if cfg == 1:  # small enough to compare every output with the oracle
        kc, vc = oracle.caches_for(dec.w)
        want = oracle.decode_for(dec.w, kc, vc)
        got = out.float().cpu().numpy().astype(np.float64)
        max_abs = float(np.abs(got - want).max())
        rel = float(np.linalg.norm(got - want) / np.linalg.norm(want))
        assert max_abs <= MAX_ABS and rel <= REL_L2, (max_abs, rel)


def test_static_scratch_small_call_after_a_large_one():
    """Config 4 (long contexts, 64 partitions a row) fills most of the array;
    config 1 then reuses its start.  Both must equal the workspace entry point
    bit for bit, the second one included."""
    import paged_kv_cache_369_b200 as pa

    P = 512
    big, big_ref = _decoder(4, P)
    small, small_ref = _decoder(1, P)
    _static_twice(pa, big, big_ref, P)
    _static_twice(pa, small, small_ref, P)
    _static_twice(pa, big, big_ref, P)


def test_static_scratch_rejects_sizes_beyond_its_array():
    import paged_kv_cache_369_b200 as pa

    S, Hq, d, L, P = 1024, 64, 128, 32768, 512
    assert pa.pa_split_workspace_bytes(S, Hq, d, L, P) > pa.PA_STATIC_SCRATCH_BYTES
    dummy = 1 << 20  # never dereferenced: the size check comes first
    status = pa.lib().pa_decode_split_reduce_static_scratch(
        dummy, dummy, dummy, dummy, dummy, L // 16, dummy, S, Hq, 8, d, 16, 100000, 0.088,
        pa.PA_BF16, pa.PA_BF16, 1.0, 1.0, P, L, None, None)
    assert status == pa.PA_ERR_INVALID_ARG
