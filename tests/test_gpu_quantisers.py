"""The device quantisers of the 8-bit caches at their edge cases, byte for
byte against the oracle.

The 8-bit formats and their ranges are fixed by the pages: FP8 E4M3 with
largest value 448 and E5M2 with 57344 ("大语言模型推理引擎深度剖析：从 KV Cache
内存管理到 PagedAttention、投机解码与量化加速的完全工程指南", §4.2-§4.3), INT8 beside
them (openeuler page, §2.3).  Every path that stores codes -- pa_cache_write,
pa_cache_write_per_channel and the store inside pa_decode_append's attention
launch (and its CUDA-core append kernel) -- is fed:

  - every one of the 2^16 f16 and the 2^16 bf16 bit patterns (so +-0,
    subnormals, +-Inf and every NaN payload are all there);
  - inputs that land exactly on a rounding tie of the format: the midpoint of
    every pair of adjacent codes (and of the largest code and the next step
    beyond it), times a power-of-two scale, positive and negative;

under several scales: 1, a power of two small enough that most inputs
saturate, non-powers of two, and one large enough that most inputs round to
zero or into the subnormal codes.  The pools (poison bytes included) must equal
the oracle's bit for bit.
"""

import numpy as np
import pytest
import torch

import oracle
import workload

pytestmark = pytest.mark.gpu

ALL16 = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)

# (name, scale); the saturating power of two puts the format's largest code
# at an input magnitude of about 0.4 (E4M3, INT8) or 0.05 (E5M2)
SCALES = {
    "e4m3": [1.0, 2.0 ** -10, 0.3, 146.21875, 1.7e-3, 2.0 ** 9 * 1.37],
    "e5m2": [1.0, 2.0 ** -20, 0.3, 1.1423, 3.3e-6, 2.0 ** 12 * 1.37],
    "int8": [1.0, 2.0 ** -10, 0.3, 515.77, 7.9e-3, 2.0 ** 9 * 1.37],
}


def _pa():
    import paged_kv_cache_369_b200 as pa
    from paged_kv_cache_369_b200.runner import PagedDecode

    return pa, PagedDecode


def _code_values(kv: str) -> np.ndarray:
    """Sorted distinct finite non-negative values of the format's codes,
    decoded by the oracle."""
    vals = oracle.decode_bits(np.arange(256, dtype=np.uint8), kv)
    vals = vals[np.isfinite(vals) & (vals >= 0)]
    return np.unique(vals)


def tie_inputs(kv: str, act: str, scale_pow2: float) -> np.ndarray:
    """16-bit patterns x with x / scale exactly halfway between two adjacent
    codes (and halfway past the largest one), for a power-of-two scale;
    both signs.  Only midpoints the activation format holds exactly are
    kept."""
    v = _code_values(kv)
    step = v[-1] - v[-2]
    mids = np.concatenate([(v[:-1] + v[1:]) / 2, [v[-1] + step / 2]])
    x = np.concatenate([mids, -mids]) * scale_pow2
    bits = workload.f32_to_bits(x.astype(np.float32), act)
    exact = workload.bits_to_f32(bits, act).astype(np.float64) == x
    assert exact.mean() > 0.95, (kv, act, exact.mean())
    return bits[exact]


def edge_inputs(kv: str, act: str) -> np.ndarray:
    """All 2^16 patterns, then the ties at scales 1 and 2^-3."""
    return np.concatenate([ALL16, tie_inputs(kv, act, 1.0), tie_inputs(kv, act, 0.125)])


def rows_of(bits: np.ndarray, hk: int, d: int, roll: int = 0) -> np.ndarray:
    """Lay a flat pattern list out as [T, Hk, d] token rows (zero padded)."""
    per = hk * d
    T = -(-bits.size // per)
    flat = np.zeros(T * per, dtype=np.uint16)
    flat[:bits.size] = np.roll(bits, roll)
    return flat.reshape(T, hk, d)


def _dev16(a: np.ndarray, act: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16))
    return t.view(torch.float16 if act == "f16" else torch.bfloat16).cuda()


def _pools(pa, nb, hk, B, d, kv):
    dt = pa.pool_torch_dtype(kv)
    kc = torch.empty((nb, hk, B, d), dtype=dt, device="cuda")
    vc = torch.empty_like(kc)
    kc.view(torch.uint8).fill_(0xFF)
    vc.view(torch.uint8).fill_(0xFF)
    return kc, vc


def _bytes(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.uint8).cpu().numpy()


def _assert_pool_equal(gpu: torch.Tensor, ref: np.ndarray, what: str):
    g = _bytes(gpu).reshape(-1)
    r = ref.view(np.uint8).reshape(-1)
    bad = np.nonzero(g != r)[0]
    assert bad.size == 0, f"{what}: {bad.size} bytes differ, first at {bad[:4]} gpu {g[bad[:4]]} oracle {r[bad[:4]]}"


def _scattered_slots(T: int, nb: int, B: int, seed: int) -> np.ndarray:
    """T distinct slots spread over a pool of nb blocks (slot = block * B + offset)."""
    return np.random.default_rng(seed).permutation(nb * B)[:T].astype(np.int64)


@pytest.mark.parametrize("scale_i", range(6))
@pytest.mark.parametrize("kv", ["e4m3", "e5m2", "int8"])
@pytest.mark.parametrize("act", ["f16", "bf16"])
def test_cache_write_quantiser_edges(act, kv, scale_i):
    """pa_cache_write over every 16-bit pattern and every tie, K and V."""
    pa, _ = _pa()
    hk, d, B = 2, 128, 16
    k_scale = float(np.float32(SCALES[kv][scale_i]))
    v_scale = float(np.float32(SCALES[kv][(scale_i + 1) % 6]))
    bits = edge_inputs(kv, act)
    kr = rows_of(bits, hk, d)
    vr = rows_of(bits, hk, d, roll=777)  # V sees the same inputs at other positions
    T = kr.shape[0]
    nb = -(-T // B) + 3
    slots = _scattered_slots(T, nb, B, seed=scale_i)
    kc, vc = _pools(pa, nb, hk, B, d, kv)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_cache_write(_dev16(kr, act), _dev16(vr, act), kc, vc, torch.from_numpy(slots).cuda(),
                      k_scale, v_scale, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rk = oracle.empty_pool(nb, hk, B, d, kv)
    rv = oracle.empty_pool(nb, hk, B, d, kv)
    assert oracle.cache_write(kr, vr, rk, rv, slots, nb, hk, d, B, act, kv, k_scale, v_scale) == 0
    _assert_pool_equal(kc, rk, f"K {act}->{kv} scale {k_scale}")
    _assert_pool_equal(vc, rv, f"V {act}->{kv} scale {v_scale}")


@pytest.mark.parametrize("kv", ["e4m3", "e5m2", "int8"])
@pytest.mark.parametrize("act", ["f16", "bf16"])
def test_cache_write_per_channel_quantiser_edges(act, kv):
    """pa_cache_write_per_channel: every channel gets one of the scales above
    (cycled, so each scale meets every input position over the rows)."""
    pa, _ = _pa()
    hk, d, B = 2, 128, 16
    sc = np.array(SCALES[kv], dtype=np.float32)
    k_chan = sc[np.arange(hk * d) % sc.size].reshape(hk, d)
    v_chan = sc[(np.arange(hk * d) * 5 + 1) % sc.size].reshape(hk, d)
    bits = edge_inputs(kv, act)
    # repeat the inputs with a shift so every pattern meets several scales
    kr = np.concatenate([rows_of(bits, hk, d, roll=r) for r in (0, 1, 2)])
    vr = np.concatenate([rows_of(bits, hk, d, roll=r) for r in (3, 4, 5)])
    T = kr.shape[0]
    nb = -(-T // B) + 2
    slots = _scattered_slots(T, nb, B, seed=11)
    kc, vc = _pools(pa, nb, hk, B, d, kv)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_cache_write_per_channel(_dev16(kr, act), _dev16(vr, act), kc, vc,
                                  torch.from_numpy(slots).cuda(), torch.from_numpy(k_chan).cuda(),
                                  torch.from_numpy(v_chan).cuda(), err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rk = oracle.empty_pool(nb, hk, B, d, kv)
    rv = oracle.empty_pool(nb, hk, B, d, kv)
    assert oracle.cache_write_channel(kr, vr, rk, rv, slots, nb, hk, d, B, act, kv, k_chan,
                                      v_chan) == 0
    _assert_pool_equal(kc, rk, f"K per-channel {act}->{kv}")
    _assert_pool_equal(vc, rv, f"V per-channel {act}->{kv}")


@pytest.mark.parametrize("kernel", ["auto", "simt"])
@pytest.mark.parametrize("mode", ["fused", "fused_single"])
@pytest.mark.parametrize("kv", ["e4m3", "e5m2", "int8"])
@pytest.mark.parametrize("act", ["f16", "bf16"])
def test_append_store_quantiser_edges(act, kv, mode, kernel, monkeypatch):
    """pa_decode_append: the attention launch stores each sequence's new token
    (tensor-core kernel, through its own swizzled tile write) or, with the
    CUDA-core kernel, the append kernel does; the new rows carry every edge
    input.  The earlier tokens are ordinary draws written by pa_cache_write.
    Pools must equal the oracle's; the attention output is not compared (it
    sees NaN and saturated inputs) but must raise no device error."""
    if kernel == "simt":
        monkeypatch.setenv("PA369_DECODE_KERNEL", "simt")
    else:
        monkeypatch.delenv("PA369_DECODE_KERNEL", raising=False)
    pa, PagedDecode = _pa()
    hk, d = 8, 128
    bits = edge_inputs(kv, act)
    kn = rows_of(bits, hk, d)
    S = kn.shape[0]
    vn = rows_of(bits, hk, d, roll=4099)
    lens = (np.arange(S) * 7) % 40 + 1  # new token at positions 0 .. 39, all tile offsets
    w = workload.build(f"q8 append {act} {kv}", 7100, lens, 4 * hk, hk, d, act, kv,
                       extra_table_cols=1)
    w.k_new, w.v_new = kn, vn
    # the saturating scale for K, a non-power of two for V (the prefill rows
    # are N(0, 1) draws quantised with the same scales)
    w.k_scale = float(np.float32(SCALES[kv][1]))
    w.v_scale = float(np.float32(SCALES[kv][2]))
    dec = PagedDecode(w, mode=mode, partition_size=16)
    dec.step()
    torch.cuda.synchronize()
    assert dec.error() == 0
    kc, vc = oracle.caches_for(w)
    _assert_pool_equal(dec.k_cache, kc, f"K append {act}->{kv} {mode} {kernel}")
    _assert_pool_equal(dec.v_cache, vc, f"V append {act}->{kv} {mode} {kernel}")
