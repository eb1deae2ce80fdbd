"""The C ABI without a GPU: the library loads, exports every symbol that
include/pa.h declares, and its host-side checks reject bad arguments with the
documented status before any CUDA call."""

import ctypes
import os
import re
import subprocess

import pytest

from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "pa.h")


@pytest.fixture(scope="module")
def pa():
    import importlib.util

    spec = importlib.util.spec_from_file_location(
        "_pa369_build", os.path.join(ROOT, "paged_kv_cache_369_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    b.build()
    import paged_kv_cache_369_b200 as m

    return m


def header_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = header_symbols()
    for s in ("pa_slot_mapping", "pa_cache_write", "pa_decode", "pa_decode_split_reduce",
              "pa_split_workspace_bytes", "pa_status_string"):
        assert s in syms


def test_library_exports_every_header_symbol(pa):
    out = subprocess.run(["nm", "-D", "--defined-only", pa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (pa_[a-z_0-9]+)\b", out))
    missing = [s for s in header_symbols() if s not in exported]
    assert not missing, f"declared but not exported: {missing}"
    lib = ctypes.CDLL(pa.LIB_PATH)
    for s in header_symbols():
        assert hasattr(lib, s)
    assert sorted(pa.SYMBOLS) == sorted(header_symbols())


def test_status_strings(pa):
    for code in range(6):
        assert pa.pa_status_string(code).startswith("PA_")
    assert pa.pa_status_string(99) == "unknown pa_status"
    assert pa.pa_version() == 10000


A = 1 << 20  # a 16-byte aligned non-null stand-in pointer; never dereferenced


def _decode(pa, **kw):
    args = dict(out=A, q=A, k=A, v=A, bt=A, mbs=4, sl=A, S=2, Hq=8, Hk=2, d=128, B=16, NB=10,
                scale=0.1, qd=pa.PA_BF16, kvd=pa.PA_BF16, ks=1.0, vs=1.0)
    args.update(kw)
    return pa.lib().pa_decode(args["out"], args["q"], args["k"], args["v"], args["bt"],
                              args["mbs"], args["sl"], args["S"], args["Hq"], args["Hk"],
                              args["d"], args["B"], args["NB"], args["scale"], args["qd"],
                              args["kvd"], args["ks"], args["vs"], None, None)


@pytest.mark.parametrize("kw,status", [
    (dict(d=96), 2),                                  # head_dim
    (dict(d=256), 2),
    (dict(B=64), 2),                                  # block size (16 or 32)
    (dict(B=8), 2),
    (dict(Hq=8, Hk=3), 1),                            # Hq % Hk
    (dict(Hk=0), 1),
    (dict(qd=2), 2),                                  # fp8 query
    (dict(qd=0, kvd=1), 2),                           # f16 q with bf16 cache
    (dict(q=0), 1),                                   # null pointers
    (dict(out=0), 1),
    (dict(bt=0), 1),
    (dict(sl=0), 1),
    (dict(k=A + 8), 1),                               # misaligned
    (dict(out=A + 2), 1),
    (dict(NB=0), 1),
    (dict(mbs=0), 1),
    (dict(scale=float("inf")), 1),
    (dict(kvd=2, ks=0.0), 1),                         # fp8 needs positive scales
    (dict(kvd=2, vs=float("nan")), 1),
    (dict(S=-1), 1),
])
def test_decode_rejects(pa, kw, status):
    assert _decode(pa, **kw) == status


def test_decode_empty_batch_is_a_noop(pa):
    assert _decode(pa, S=0, q=0, out=0) == 0


def test_split_checks(pa):
    L = pa.lib()
    need = pa.pa_split_workspace_bytes(2, 8, 128, 1000, 512)
    assert need == 256 + (2 * 8 * 2 * 128 * 4 + 255) // 256 * 256
    assert pa.pa_split_workspace_bytes(2, 8, 128, 1000, 0) == 0

    def call(P=512, maxlen=1000, ws=A, wsb=need):
        return L.pa_decode_split_reduce(A, A, A, A, A, 4, A, 2, 8, 2, 128, 16, 10, 0.1,
                                        pa.PA_BF16, pa.PA_BF16, 1.0, 1.0, P, maxlen, ws, wsb,
                                        None, None)

    assert call(P=24) == 1            # not a multiple of the block size
    assert call(P=0) == 1
    assert call(maxlen=-1) == 1
    assert call(wsb=need - 1) == 1    # workspace too small
    assert call(ws=0) == 1
    assert call(ws=A + 128) == 1      # workspace must be 256-byte aligned
    assert call(P=(1 << 30) + 16) == 1                     # partitions of at most 2^30 tokens
    assert call(maxlen=(1 << 30) + 1) == 1                 # max_seq_len at most 2^30
    # near the int range the partition count is still exact (no overflow):
    # ceil((2^31 - 1) / 2^30) = 2 partitions
    big = pa.pa_split_workspace_bytes(1, 1, 64, (1 << 31) - 1, 1 << 30)
    assert big == 256 + 2 * 64 * 4


def test_static_scratch_checks_arguments_before_the_device(pa):
    """The allocation-free split entry point returns the argument errors of
    pa_decode_split_reduce without touching the GPU (none here), so they never
    turn into PA_ERR_CUDA."""
    L = pa.lib()

    def call(S=2, Hq=8, Hk=2, d=128, P=512, maxlen=1000, scale=0.1, kvd=None, out=A):
        return L.pa_decode_split_reduce_static_scratch(
            out, A, A, A, A, 4, A, S, Hq, Hk, d, 16, 10, scale, pa.PA_BF16,
            pa.PA_BF16 if kvd is None else kvd, 1.0, 1.0, P, maxlen, None, None)

    assert call(Hq=0) == 1
    assert call(Hq=6, Hk=4) == 1      # not a whole GQA group
    assert call(P=0) == 1
    assert call(P=24) == 1
    assert call(maxlen=-1) == 1
    assert call(scale=float("nan")) == 1
    assert call(out=A + 8) == 1       # misaligned
    assert call(d=96) == 2            # unsupported head_dim
    assert call(kvd=pa.PA_F16) == 2   # 16-bit cache of another dtype
    assert call(S=0) == 0             # empty batch: nothing to do, no device needed
    # too large for the built-in array (checked before the device as well)
    assert call(S=1024, Hq=64, Hk=8, maxlen=32768) == 1


def test_cache_write_and_slot_checks(pa):
    L = pa.lib()
    cw = lambda **k: L.pa_cache_write(k.get("kn", A), A, k.get("kc", A), A, k.get("sm", A),
                                      k.get("T", 4), 10, 2, k.get("d", 128), 16,
                                      k.get("act", pa.PA_BF16), k.get("kv", pa.PA_BF16),
                                      k.get("ks", 1.0), 1.0, None, None)
    assert cw(act=pa.PA_FP8_E4M3) == 2
    assert cw(act=pa.PA_F16, kv=pa.PA_BF16) == 2
    assert cw(d=12) == 2
    assert cw(kv=pa.PA_FP8_E4M3, ks=-1.0) == 1
    assert cw(kn=0) == 1
    assert cw(kc=A + 4) == 1
    assert cw(T=-1) == 1
    assert cw(T=0, kn=0) == 0
    sm = lambda **k: L.pa_slot_mapping(k.get("out", A), k.get("bt", A), k.get("mbs", 4),
                                       k.get("sl", A), k.get("ts", None), k.get("tp", None),
                                       k.get("T", 2), k.get("S", 2), 16, 10, None, None)
    assert sm(out=0) == 1
    assert sm(bt=0) == 1
    assert sm(mbs=0) == 1
    assert sm(sl=None) == 1           # decode form needs seq_lens
    assert sm(T=3, S=2) == 1          # token t is sequence t: T <= S
    assert sm(T=0, out=0) == 0


def test_decode_append_checks(pa):
    L = pa.lib()

    def call(kn=A, vn=A, P=512, ws=A, wsb=1 << 30, maxlen=1000, S=2):
        return L.pa_decode_append(A, A, kn, vn, A, A, A, 4, A, S, 8, 2, 128, 16, 10, 0.1,
                                  pa.PA_BF16, pa.PA_BF16, 1.0, 1.0, P, maxlen, ws, wsb, None, None)

    assert call(kn=0) == 1            # new rows required
    assert call(vn=A + 8) == 1        # misaligned
    assert call(P=24) == 1            # partition not a multiple of 16
    assert call(P=-16) == 1
    assert call(ws=0) == 1            # split needs a workspace
    assert call(wsb=16) == 1
    assert call(S=0, kn=0) == 0       # empty batch


def test_copy_blocks_checks(pa):
    L = pa.lib()

    def call(k=A, v=A, pairs=A, n=3, nb=10, hk=2, d=128, kv=pa.PA_BF16):
        return L.pa_copy_blocks(k, v, pairs, n, nb, hk, d, 16, kv, None, None)

    assert call(n=-1) == 1
    assert call(nb=0) == 1
    assert call(hk=0) == 1
    assert call(kv=7) == 2            # unknown element type
    assert call(pairs=0) == 1
    assert call(k=0) == 1
    assert call(v=A + 8) == 1         # misaligned pool
    assert call(n=0, pairs=0, k=0, v=0) == 0   # nothing to copy


def test_prefill_checks(pa):
    L = pa.lib()

    def call(out=A, q=A, qs=A, S=2, T=8, mq=4, Hq=8, Hk=2, d=128, B=16, NB=10, qd=pa.PA_BF16,
             kvd=pa.PA_BF16, scale=0.1, ks=1.0, vs=1.0):
        return L.pa_prefill(out, q, A, A, A, 4, A, qs, S, T, mq, Hq, Hk, d, B, NB, scale, qd, kvd,
                            ks, vs, None, None)

    assert call(kvd=pa.PA_FP8_E4M3, d=64) == 2   # 8-bit caches: head_dim 128
    assert call(kvd=pa.PA_FP8_E4M3, ks=0.0) == 1  # 8-bit caches need positive scales
    assert call(kvd=pa.PA_INT8, vs=float("inf")) == 1
    assert call(qd=pa.PA_F16) == 2           # cache dtype must be the q dtype
    assert call(d=96) == 2
    assert call(B=64) == 2
    assert call(Hq=8, Hk=3) == 1
    assert call(Hq=256, Hk=1) == 2           # group above 128
    assert call(qs=0) == 1
    assert call(out=A + 4) == 1
    assert call(mq=0) == 1
    assert call(S=-1) == 1
    assert call(scale=float("nan")) == 1
    assert call(scale=-0.5) == 1             # the softmax scale must be positive
    assert call(S=0, q=0) == 0               # nothing to do
    assert call(T=0, q=0) == 0


def test_per_channel_checks(pa):
    L = pa.lib()

    def cw(kv=pa.PA_FP8_E4M3, ks=A, vs=A, T=4):
        return L.pa_cache_write_per_channel(A, A, A, A, A, T, 10, 2, 128, 16, pa.PA_BF16, kv, ks,
                                            vs, None, None)

    assert cw(kv=pa.PA_BF16) == 2           # per-channel scales need an 8-bit cache
    assert cw(ks=0) == 1
    assert cw(vs=A + 4) == 1                 # scales read as 16-byte vectors
    assert cw(T=0, ks=0) == 0

    def dec(kv=pa.PA_FP8_E4M3, ks=A, vs=A, P=0, ws=None, wsb=0, S=2):
        return L.pa_decode_per_channel(A, A, A, A, A, 4, A, S, 8, 2, 128, 16, 10, 0.1, pa.PA_BF16,
                                       kv, ks, vs, P, 1000, ws, wsb, None, None)

    assert dec(kv=pa.PA_BF16) == 2
    assert dec(ks=0) == 1
    assert dec(vs=A + 2) == 1
    assert dec(P=24) == 1
    assert dec(P=512) == 1                   # split needs a workspace
    assert dec(S=0) == 0                     # empty batch


def test_shared_prefix_checks(pa):
    L = pa.lib()
    need = pa.pa_shared_prefix_workspace_bytes(2, 8, 128, 1000, 512, 256)
    # 2 prefix key ranges (ceil(512 / 256)) + ceil(488 / 256) = 2 tail partitions
    assert need == 256 + (2 * 8 * 4 * 128 * 4 + 255) // 256 * 256

    def slots(prefix, max_len, P=256):  # workspace slots per (sequence, head)
        b = pa.pa_shared_prefix_workspace_bytes(1, 1, 64, max_len, prefix, P)
        return (b - 256) // (64 * 4)

    assert slots(16, 16) == 1                 # one key tile: one range, no tail
    assert slots(256, 256) == 1
    assert slots(1024, 1024) == 4             # 16 tiles in 4 ranges of 4
    assert slots(1024, 1024 + 300) == 4 + 2
    assert slots(4096, 4096) == 8             # at most 8 ranges
    assert slots(320, 320) == 2               # 5 tiles: ranges of 3 and 2
    assert pa.pa_shared_prefix_workspace_bytes(2, 8, 128, 1000, 512, 0) == 0

    def call(prefix=512, P=256, kv=pa.PA_BF16, ws=A, wsb=need, maxlen=1000, B=16, scale=0.1,
             ks=1.0, d=128):
        return L.pa_decode_shared_prefix(A, A, A, A, A, 80, A, 2, 8, 2, d, B, 10, scale,
                                         pa.PA_BF16, kv, ks, 1.0, prefix, P, maxlen, ws, wsb, None,
                                         None)

    assert call(kv=pa.PA_FP8_E4M3, d=64) == 2   # 8-bit caches: head_dim 128
    assert call(kv=pa.PA_FP8_E4M3, ks=-1.0) == 1
    assert call(prefix=0) == 1
    assert call(prefix=24) == 1              # not a multiple of the block size
    assert call(prefix=1200) == 1            # longer than max_seq_len
    assert call(P=24) == 1
    assert call(wsb=need - 1) == 1
    assert call(ws=A + 64) == 1
    assert call(scale=-1.0) == 1
