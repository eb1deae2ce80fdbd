"""Failure detection on the GPU without a fault: a bounded device wait that
runs out reports PA_ERR_DEVICE_TIMEOUT through dev_err, the outputs stay
finite, and the context stays usable (a normal call right after it matches
the oracle).

The wait is made to run out through the decode kernels' test hook
(environment variable PA369_TEST_DECODE_STALL_NS, read by the C shim on every
decode call): every warp leaves its first tile's copies unissued, so its first
wait can only give up, after the given number of nanoseconds.  The copies the
warp did issue are drained (with their own bound) before the CTA moves on, so
no copy is in flight when it exits.  Nothing here faults, traps or hangs the
GPU: every wait ends by itself."""

import numpy as np
import pytest
import torch

import oracle
import workload
from tests.test_gpu_parity import assert_close

pytestmark = pytest.mark.gpu

STALL_NS = "200000"  # 200 us per timed-out wait


def _pa():
    import paged_kv_cache_369_b200 as pa
    from paged_kv_cache_369_b200.runner import PagedDecode

    return pa, PagedDecode


@pytest.mark.parametrize("kernel", ["auto", "simt"])
@pytest.mark.parametrize("mode,P,chain", [("single", 512, None), ("split", 64, None), ("fused", 64, None),
                                          ("split", 32, "2"), ("fused", 32, "1")])
def test_decode_wait_timeout_is_reported(mode, P, chain, kernel, monkeypatch):
    """With 32-token partitions (22 for the longest sequence) the
    tensor-core kernel's warps take 2 (or 1) partitions in a row
    (PA369_DECODE_CHAIN)."""
    if chain:
        monkeypatch.setenv("PA369_DECODE_CHAIN", chain)
    if kernel == "simt":
        monkeypatch.setenv("PA369_DECODE_KERNEL", "simt")
    else:
        monkeypatch.delenv("PA369_DECODE_KERNEL", raising=False)
    pa, PagedDecode = _pa()
    w = workload.build("timeout", 6100, [1, 40, 300, 700], 16, 4, 128, "bf16", "bf16",
                       extra_table_cols=1)
    kc, vc = oracle.caches_for(w)
    ref = oracle.decode_for(w, kc, vc)
    dec = PagedDecode(w, mode=mode, partition_size=P)
    dec.step()
    torch.cuda.synchronize()
    assert dec.error() == 0
    assert_close(dec.out.float().cpu().numpy().astype(np.float64), ref, "before the timeout")

    # every warp's first wait runs out
    monkeypatch.setenv("PA369_TEST_DECODE_STALL_NS", STALL_NS)
    dec.dev_err.zero_()
    dec.out.fill_(float("nan"))
    dec.step() if mode == "fused" else dec.attend()
    torch.cuda.synchronize()
    assert dec.error() == pa.PA_ERR_DEVICE_TIMEOUT
    assert torch.isfinite(dec.out.float()).all()

    # the hook off again: the same process and context give the right answer
    monkeypatch.delenv("PA369_TEST_DECODE_STALL_NS")
    dec.dev_err.zero_()
    dec.attend()
    torch.cuda.synchronize()
    assert dec.error() == 0
    assert_close(dec.out.float().cpu().numpy().astype(np.float64), ref, "after the timeout")


def test_timeout_then_other_kernels_still_run(monkeypatch):
    """After a timed-out decode, the cache write and a chunked prefill on the
    same context still match the oracle."""
    pa, PagedDecode = _pa()
    from paged_kv_cache_369_b200.runner import PagedPrefill

    w = workload.build("timeout2", 6101, [33, 129], 8, 2, 64, "f16", "f16")
    dec = PagedDecode(w, mode="split", partition_size=32)
    monkeypatch.setenv("PA369_TEST_DECODE_STALL_NS", STALL_NS)
    dec.step()
    torch.cuda.synchronize()
    assert dec.error() == pa.PA_ERR_DEVICE_TIMEOUT
    monkeypatch.delenv("PA369_TEST_DECODE_STALL_NS")
    kc, vc = oracle.caches_for(w)  # the cache write of the step itself was not affected
    assert np.array_equal(dec.k_cache.view(torch.uint8).cpu().numpy(), kc.view(np.uint8).reshape(
        dec.k_cache.view(torch.uint8).shape))
    pw = workload.build_chunked("after timeout", 6102, [5, 40], [20, 33], 8, 2, 128, "bf16", "bf16")
    pre = PagedPrefill(pw)
    pre.step()
    torch.cuda.synchronize()
    assert pre.error() == 0
    pkc, pvc = oracle.chunked_caches_for(pw)
    assert_close(pre.out.float().cpu().numpy().astype(np.float64),
                 oracle.prefill_for(pw, pkc, pvc), "prefill after a timeout")


@pytest.mark.parametrize("kv", ["bf16", "e4m3"])
def test_prefill_wait_timeout_is_reported(kv, monkeypatch):
    """The chunked prefill's abort path: with PA369_TEST_PREFILL_STALL_NS set
    (read by the launch), every CTA leaves its first K/V stage's copies
    unissued, so the wait on that stage runs out; the role that gives up raises
    the CTA's abort flag, every other role leaves its own bounded wait, the
    copies that were issued are drained and TMEM is freed.  The launch reports
    PA_ERR_DEVICE_TIMEOUT, and a normal prefill on the same context right after
    matches the oracle."""
    pa, _ = _pa()
    from paged_kv_cache_369_b200.runner import PagedPrefill

    w = workload.build_chunked("prefill timeout", 6103, [5, 300], [40, 200], 16, 4, 128, "bf16", kv)
    pkc, pvc = oracle.chunked_caches_for(w)
    ref = oracle.prefill_for(w, pkc, pvc)
    pre = PagedPrefill(w)
    pre.step()
    torch.cuda.synchronize()
    assert pre.error() == 0
    assert_close(pre.out.float().cpu().numpy().astype(np.float64), ref, "prefill before the timeout")

    monkeypatch.setenv("PA369_TEST_PREFILL_STALL_NS", STALL_NS)
    pre.dev_err.zero_()
    pre.attend()
    torch.cuda.synchronize()
    assert pre.error() == pa.PA_ERR_DEVICE_TIMEOUT

    monkeypatch.delenv("PA369_TEST_PREFILL_STALL_NS")
    pre.dev_err.zero_()
    pre.out.fill_(float("nan"))
    pre.attend()
    torch.cuda.synchronize()
    assert pre.error() == 0
    assert_close(pre.out.float().cpu().numpy().astype(np.float64), ref, "prefill after the timeout")
