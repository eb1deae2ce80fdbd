"""Pins for the oracle's other 8-bit KV formats (openeuler page §2.3 lists
FP8 E5M2 / E4M3 and INT8 KV caches; the fifth page's §4.2 gives the E5M2
range): the E5M2 decoder and encoder against torch's float8_e5m2, the
saturation bound printed on the page, INT8 against numpy's round-half-even
and clip, and decode attention on both formats against torch SDPA on
values dequantised by torch / numpy."""

import json
import math
import os

import numpy as np
import pytest
import torch

import workload
from tests.test_oracle_pins import _contiguous_kv, _sdpa_ref


def _torch_e5m2(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e5m2).double().numpy()


def test_e5m2_decode_all_codes_vs_torch(orc):
    codes = np.arange(256, dtype=np.uint8)
    ref = _torch_e5m2(codes)
    got = np.array([orc.e5m2_decode(int(c)) for c in codes])
    assert np.array_equal(np.isnan(ref), np.isnan(got)) and np.isnan(got).sum() == 6
    m = ~np.isnan(ref)
    assert np.array_equal(ref[m], got[m])
    assert np.isinf(got).sum() == 2


def test_e5m2_range_printed(orc, golden_dir):
    with open(os.path.join(golden_dir, "fp8_ranges.json")) as f:
        g = json.load(f)["e5m2"]
    finite = [orc.e5m2_decode(c) for c in range(256) if math.isfinite(orc.e5m2_decode(c))]
    assert max(finite) == g["max_abs"] and min(finite) == -g["max_abs"]
    # satfinite: overflow and infinity clamp to the largest finite code
    for y, code in ((1e30, 0x7B), (-1e30, 0xFB), (float("inf"), 0x7B), (57344.0, 0x7B),
                    (61439.0, 0x7B), (-float("inf"), 0xFB)):
        assert orc.e5m2_encode(y) == code
    assert orc.e5m2_encode(float("nan")) == 0x7F


def test_e5m2_encode_identity_and_midpoints_vs_torch(orc):
    for c in range(256):
        v = orc.e5m2_decode(c)
        if math.isfinite(v) and not (v == 0 and c == 0x80):
            assert orc.e5m2_encode(v) == c, hex(c)
    vals = sorted({orc.e5m2_decode(c) for c in range(0x7C)})
    mids = [(a + b) / 2 for a, b in zip(vals, vals[1:])]
    ys = np.array(mids + [-m for m in mids], dtype=np.float32)
    rng = np.random.default_rng(12)
    ys = np.concatenate([ys, (rng.standard_normal(30000) * 3000).astype(np.float32)])
    ys = ys[np.abs(ys) < 57344]
    ref = torch.from_numpy(ys).to(torch.float8_e5m2).view(torch.uint8).numpy()
    got = np.array([orc.e5m2_encode(float(y)) for y in ys], dtype=np.uint8)
    assert np.array_equal(got, ref)


def test_int8_codec_vs_numpy(orc):
    rng = np.random.default_rng(13)
    ys = np.concatenate([np.arange(-130, 131, 0.5), rng.standard_normal(20000) * 60]).astype(np.float32)
    ref = np.clip(np.rint(ys.astype(np.float64)), -127, 127).astype(np.int8).view(np.uint8)
    got = np.array([orc.int8_encode(float(y)) for y in ys], dtype=np.uint8)
    assert np.array_equal(got, ref)
    for c in range(256):
        assert orc.int8_decode(c) == float(np.uint8(c).view(np.int8))


@pytest.mark.parametrize("kv", ["e5m2", "int8"])
def test_cache_write_8bit_vs_library_quantiser(orc, kv):
    """Codes = library quantiser of (x / scale) computed in fp32 (torch's
    e5m2 cast; numpy rint + clip for INT8), for in-range values."""
    rng = np.random.default_rng(14)
    T, Hk, d, nb = 40, 2, 32, 8
    x = rng.standard_normal((T, Hk, d)).astype(np.float32) * 3
    bits = workload.f32_to_bits(x, "bf16")
    xf = workload.bits_to_f32(bits, "bf16")
    scale = workload.gen.per_tensor_scale(float(np.abs(xf).max()), kv)
    y = xf / np.float32(scale)
    if kv == "e5m2":
        ref = torch.from_numpy(y).to(torch.float8_e5m2).view(torch.uint8).numpy()
    else:
        ref = np.clip(np.rint(y.astype(np.float64)), -127, 127).astype(np.int8).view(np.uint8)
    slots = rng.choice(nb * 16, size=T, replace=False).astype(np.int64)
    kc = orc.empty_pool(nb, Hk, 16, d, kv)
    vc = orc.empty_pool(nb, Hk, 16, d, kv)
    orc.cache_write(bits, bits, kc, vc, slots, nb, Hk, d, 16, "bf16", kv, scale, scale)
    for t in range(T):
        b, o = divmod(int(slots[t]), 16)
        np.testing.assert_array_equal(kc[b, :, o, :], ref[t])


@pytest.mark.parametrize("kv", ["e5m2", "int8"])
def test_decode_8bit_vs_torch_sdpa_on_dequantised(orc, kv):
    w = workload.build("pin8b", 6, [9, 40, 23], 8, 2, 32, "bf16", kv)
    kc, vc = orc.caches_for(w)
    got = orc.decode_for(w, kc, vc)
    K, V = _contiguous_kv(w)
    dec = (lambda a: _torch_e5m2(a)) if kv == "e5m2" else \
        (lambda a: np.asarray(a, np.uint8).view(np.int8).astype(np.float64))
    for s in range(w.num_seqs):
        for t in range(int(w.seq_lens[s])):
            phys, off = w.block_tables[s, t // 16], t % 16
            K[s][t] = dec(kc[phys, :, off, :]) * w.k_scale
            V[s][t] = dec(vc[phys, :, off, :]) * w.v_scale
    ref = _sdpa_ref(w, K, V)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# per-channel scales (the fifth page's §4.3: each channel of K / V quantised
# separately)
# ---------------------------------------------------------------------------

def test_cache_write_per_channel_vs_torch_quantiser(orc):
    """Codes = torch's e4m3fn cast of (x / s[h][i]) computed in fp32."""
    rng = np.random.default_rng(15)
    T, Hk, d, nb = 40, 3, 32, 8
    x = (rng.standard_normal((T, Hk, d)) * rng.uniform(0.1, 8.0, size=(1, Hk, d))).astype(np.float32)
    bits = workload.f32_to_bits(x, "bf16")
    xf = workload.bits_to_f32(bits, "bf16")
    sc = workload.gen.per_channel_scales("e4m3", bits, dtype="bf16")
    assert sc.shape == (Hk, d) and sc.dtype == np.float32
    ref = torch.from_numpy(xf / sc[None]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    slots = rng.choice(nb * 16, size=T, replace=False).astype(np.int64)
    kc = orc.empty_pool(nb, Hk, 16, d, "e4m3")
    vc = orc.empty_pool(nb, Hk, 16, d, "e4m3")
    orc.cache_write_channel(bits, bits, kc, vc, slots, nb, Hk, d, 16, "bf16", "e4m3", sc, sc)
    for t in range(T):
        b, o = divmod(int(slots[t]), 16)
        np.testing.assert_array_equal(kc[b, :, o, :], ref[t])
    # each channel's largest |x| maps onto the largest code
    assert (np.abs(ref.view(np.uint8) & 0x7F).max(axis=0) == 0x7E).all()


@pytest.mark.parametrize("kv", ["e4m3", "int8"])
def test_decode_per_channel_vs_torch_sdpa(orc, kv):
    w = workload.build("pinch", 16, [9, 40, 23], 8, 2, 32, "bf16", kv, channel_scales=True)
    kc, vc = orc.caches_for(w)
    got = orc.decode_for(w, kc, vc)
    K, V = _contiguous_kv(w)
    dec = (lambda a: torch.from_numpy(np.asarray(a, np.uint8)).view(torch.float8_e4m3fn).double().numpy()) \
        if kv == "e4m3" else (lambda a: np.asarray(a, np.uint8).view(np.int8).astype(np.float64))
    for s in range(w.num_seqs):
        for t in range(int(w.seq_lens[s])):
            phys, off = w.block_tables[s, t // 16], t % 16
            K[s][t] = dec(kc[phys, :, off, :]) * w.k_chan.astype(np.float64)
            V[s][t] = dec(vc[phys, :, off, :]) * w.v_chan.astype(np.float64)
    ref = _sdpa_ref(w, K, V)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_per_channel_with_equal_scales_is_per_tensor(orc):
    """Per-channel scales that all equal the per-tensor scale give the same
    pools and outputs bit for bit."""
    w = workload.build("eq", 17, [30, 5, 64], 8, 4, 32, "f16", "e4m3", channel_scales=True)
    w.k_chan[:] = np.float32(w.k_scale)
    w.v_chan[:] = np.float32(w.v_scale)
    kc, vc = orc.caches_for(w)
    out = orc.decode_for(w, kc, vc)
    k_chan, v_chan = w.k_chan, w.v_chan
    w.k_chan = w.v_chan = None
    kc2, vc2 = orc.caches_for(w)
    out2 = orc.decode_for(w, kc2, vc2)
    assert np.array_equal(kc, kc2) and np.array_equal(vc, vc2) and np.array_equal(out, out2)
    w.k_chan, w.v_chan = k_chan, v_chan
