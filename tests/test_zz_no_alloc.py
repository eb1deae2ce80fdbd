"""The allocation-free split-KV entry point against the workspace one.

pa_decode_split_reduce_static_scratch serves callers that cannot allocate
device memory (no allocator handed to them, HBM already reserved for the KV
pool, or no room for cudaMalloc's synchronisation on their path): its partials
live in a device array inside the library.  This test calls it through the C
ABI twice in a row and checks both outputs against pa_decode_split_reduce with
a caller-provided workspace, within the parity tolerance the other tests use.
It sits in its own file, collected last, and must pass alone in a fresh
process as well as after every other test (the first call on a device does the
one-time address lookup)."""

import ctypes

import numpy as np
import pytest
import torch

import workload

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
REL_L2 = 2e-3


def _close(got: torch.Tensor, ref: torch.Tensor):
    g = got.float().cpu().numpy().astype(np.float64)
    r = ref.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(g).all()
    max_abs = float(np.abs(g - r).max())
    rel = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30))
    assert max_abs <= MAX_ABS and rel <= REL_L2, (max_abs, rel)


def _call_static(pa, dec, out, P):
    w = dec.w
    return pa.lib().pa_decode_split_reduce_static_scratch(
        out.data_ptr(), dec.q.data_ptr(), dec.k_cache.data_ptr(), dec.v_cache.data_ptr(),
        dec.block_tables.data_ptr(), int(dec.block_tables.shape[1]), dec.seq_lens.data_ptr(),
        w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, w.num_blocks,
        float(w.softmax_scale), pa.dtype_code(dec.q.dtype), pa.dtype_code(dec.k_cache.dtype),
        float(w.k_scale), float(w.v_scale), P, dec.max_seq_len, dec.dev_err.data_ptr(),
        torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("cfg", [1, 2, 4])
def test_static_scratch_matches_workspace_entry_point(cfg):
    import paged_kv_cache_369_b200 as pa
    from paged_kv_cache_369_b200.runner import PagedDecode

    w = workload.config(cfg)
    P = 512
    dec = PagedDecode(w, mode="split", partition_size=P)
    dec.step()  # cache write + pa_decode_split_reduce with a torch-allocated workspace
    torch.cuda.synchronize()
    assert dec.error() == 0
    ref = dec.out.clone()
    out = torch.empty_like(ref)
    for _ in range(2):  # two calls in a row share (and reuse) the library's array
        out.fill_(float("nan"))
        status = _call_static(pa, dec, out, P)
        torch.cuda.synchronize()
        assert status == pa.PA_OK, pa.pa_status_string(status)
        assert dec.error() == 0
        _close(out, ref)


def test_static_scratch_rejects_sizes_beyond_its_array():
    import paged_kv_cache_369_b200 as pa

    S, Hq, d, L, P = 1024, 64, 128, 32768, 512
    assert pa.pa_split_workspace_bytes(S, Hq, d, L, P) > pa.PA_STATIC_SCRATCH_BYTES
    dummy = 1 << 20  # never dereferenced: the size check comes first
    status = pa.lib().pa_decode_split_reduce_static_scratch(
        dummy, dummy, dummy, dummy, dummy, L // 16, dummy, S, Hq, 8, d, 16, 100000, 0.088,
        pa.PA_BF16, pa.PA_BF16, 1.0, 1.0, P, L, None, None)
    assert status == pa.PA_ERR_INVALID_ARG
