"""Plant plausible mistakes in a copy of the oracle and check that the pins
catch every one of them.  Each mutant is built from a modified copy of
oracle.c in a temporary directory; the real oracle is never touched."""

import os
import subprocess

import numpy as np
import pytest

import oracle
from tests import test_oracle_cow as cow
from tests import test_oracle_kv_formats as kvf
from tests import test_oracle_pins as pins
from tests import test_oracle_prefill as pre

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "gqa_head_mapping_modulo": ("int kvh = h / g;", "int kvh = h % num_kv_heads;"),
    "slot_offset_from_block_index": ("return phys * block_size + pos % block_size;",
                                     "return phys * block_size + pos / block_size;"),
    "slot_block_from_offset": ("int64_t phys = block_table_row[pos / block_size];",
                               "int64_t phys = block_table_row[pos % block_size];"),
    "e4m3_bias_off_by_one": ("v = ldexp((double)(8 + m), e - 10);",
                             "v = ldexp((double)(8 + m), e - 11);"),
    "e4m3_round_half_up": ("return fmod(f, 2.0) == 0.0 ? f : f + 1.0;", "return f + 1.0;"),
    "fp8_scale_dropped_in_gather": ("rows[(int64_t)t * head_dim + i] = orc_is_8bit(kv_dtype) ? v * sc : v;",
                                    "rows[(int64_t)t * head_dim + i] = v;"),
    "softmax_scale_dropped": ("s[t] = softmax_scale * dot;", "s[t] = dot;"),
    "softmax_not_normalised": ("double p = s[t] / z;", "double p = s[t];"),
    "gather_wrong_head_stride": ("int64_t base = ((phys * num_kv_heads + kvh) * block_size + off) * head_dim;",
                                 "int64_t base = ((phys * block_size + off) * num_kv_heads + kvh) * head_dim;"),
    "split_partition_off_by_one": ("int64_t hi = lo + partition_size < len ? lo + partition_size : len;",
                                   "int64_t hi = lo + partition_size - 1 < len ? lo + partition_size - 1 : len;"),
    "lse_missing_max": ("if (lse) *lse = mx + log(z);", "if (lse) *lse = log(z);"),
    "f16_subnormal_exponent": ("v = ldexp((double)m, -24);", "v = ldexp((double)m, -25);"),
    "bf16_bias": ("v = ldexp((double)(128 + m), e - 134);", "v = ldexp((double)(128 + m), e - 133);"),
    "cache_write_skips_v": ("((uint16_t *)v_cache)[dst + i] = ((const uint16_t *)v_new)[src + i];", ""),
    "copy_blocks_k_pool_only": ("for (int pool = 0; pool < 2; ++pool) {", "for (int pool = 0; pool < 1; ++pool) {"),
    "copy_blocks_direction_swapped": (
        "base[(int64_t)dst * block_bytes + b] = base[(int64_t)src * block_bytes + b];",
        "base[(int64_t)src * block_bytes + b] = base[(int64_t)dst * block_bytes + b];"),
    "prefill_causal_off_by_one": ("qrow, K, V, pos + 1, head_dim,", "qrow, K, V, pos, head_dim,"),
    "prefill_position_from_chunk_start": ("int pos = len - n + j;", "int pos = j;"),
    "prefill_q_row_of_sequence": ("int64_t row_tok = (int64_t)query_start[s] + j;",
                                  "int64_t row_tok = (int64_t)s + j;"),
    "prefill_gqa_interleaved": ("int h = kvh * g + hh;", "int h = hh * num_kv_heads + kvh;"),
    "e5m2_bias_off_by_one": ("v = ldexp((double)(4 + m), e - 17);", "v = ldexp((double)(4 + m), e - 16);"),
    "e5m2_saturates_early": ("if (a >= 57344.0) return sign | 0x7B;", "if (a >= 49152.0) return sign | 0x7B;"),
    "int8_decoded_unsigned": ("double orc_int8_decode(uint8_t c) { return (double)(int8_t)c; }",
                              "double orc_int8_decode(uint8_t c) { return (double)c; }"),
    "e5m2_round_half_up": ("double n = orc_rne(ldexp(a, 2 - e)); /* in [4, 8] */",
                           "double n = floor(ldexp(a, 2 - e) + 0.5);"),
    "e5m2_subnormal_step": ("double n = orc_rne(a * 65536.0);", "double n = orc_rne(a * 32768.0);"),
    "int8_clamps_at_128": ("if (n > 127.0) n = 127.0;", "if (n > 128.0) n = 128.0;"),
    "int8_round_half_up": ("double n = orc_rne(fabs((double)y));", "double n = floor(fabs((double)y) + 0.5);"),
    "int8_scale_dropped_in_gather": ("rows[(int64_t)t * head_dim + i] = orc_is_8bit(kv_dtype) ? v * sc : v;",
                                     "rows[(int64_t)t * head_dim + i] = kv_dtype == ORC_E4M3 || kv_dtype == ORC_E5M2 ? v * sc : v;"),
    "channel_scale_without_head_offset": ("float yk = xk / k_scales[(int64_t)h * head_dim + i];",
                                          "float yk = xk / k_scales[i];"),
    "channel_gather_head0_scales": ("orc_gather_scaled(V, v_cache, kv_dtype, 1.0, v_scales + (int64_t)kvh * head_dim, bt, len,",
                                    "orc_gather_scaled(V, v_cache, kv_dtype, 1.0, v_scales, bt, len,"),
    "copy_blocks_one_head": ("int64_t block_bytes = (int64_t)num_kv_heads * block_size * head_dim * elem_bytes;",
                             "int64_t block_bytes = (int64_t)block_size * head_dim * elem_bytes;"),
}


def _run_pins(golden_dir):
    """Run the pin checks; return the names of the ones that failed."""
    failed = []
    checks = [
        ("worked_example", lambda: pins.test_block_table_worked_example_layout(oracle, golden_dir)),
        ("worked_example_write", lambda: pins.test_block_table_worked_example_cache_write(oracle, golden_dir)),
        ("f16", lambda: pins.test_f16_decode_exhaustive_vs_numpy(oracle)),
        ("bf16", lambda: pins.test_bf16_decode_exhaustive_vs_torch(oracle)),
        ("e4m3_decode", lambda: pins.test_e4m3_decode_all_codes_vs_torch(oracle)),
        ("e4m3_mid", lambda: pins.test_e4m3_encode_identity_and_midpoints_vs_torch(oracle)),
        ("sdpa", lambda: pins.test_decode_vs_torch_sdpa(oracle, 8, 2, 32, "bf16", [1, 16, 17, 40, 3], 0)),
        ("sdpa8", lambda: pins.test_decode_fp8_vs_torch_sdpa_on_dequantised(oracle)),
        ("closed", lambda: pins.test_closed_forms(oracle)),
        ("split", lambda: pins.test_split_equals_unsplit(oracle, 48)),
        ("roundtrip", lambda: pins.test_cache_write_then_gather_roundtrip(oracle)),
        ("prefill_sdpa", lambda: pre.test_prefill_vs_torch_sdpa_causal(
            oracle, [0, 5, 37, 16], [7, 1, 40, 16], 8, 2, 32, "bf16")),
        ("prefill_chunks", lambda: pre.test_prefill_rows_do_not_depend_on_chunking(oracle)),
        ("e5m2_decode", lambda: kvf.test_e5m2_decode_all_codes_vs_torch(oracle)),
        ("e5m2_mid", lambda: kvf.test_e5m2_encode_identity_and_midpoints_vs_torch(oracle)),
        ("e5m2_range", lambda: kvf.test_e5m2_range_printed(oracle, golden_dir)),
        ("int8", lambda: kvf.test_int8_codec_vs_numpy(oracle)),
        ("sdpa_e5m2", lambda: kvf.test_decode_8bit_vs_torch_sdpa_on_dequantised(oracle, "e5m2")),
        ("sdpa_int8", lambda: kvf.test_decode_8bit_vs_torch_sdpa_on_dequantised(oracle, "int8")),
        ("prefill_e5m2", lambda: pre.test_prefill_8bit_vs_sdpa_on_dequantised(oracle, "e5m2")),
        ("prefill_int8", lambda: pre.test_prefill_8bit_vs_sdpa_on_dequantised(oracle, "int8")),
        ("chan_write", lambda: kvf.test_cache_write_per_channel_vs_torch_quantiser(oracle)),
        ("chan_sdpa", lambda: kvf.test_decode_per_channel_vs_torch_sdpa(oracle, "e4m3")),
        ("cow_example", lambda: cow.test_cow_beam_search_example(oracle, golden_dir)),
        ("cow_brute", lambda: cow.test_copy_blocks_brute_force(oracle, "f16")),
        ("cow_bounds", lambda: cow.test_copy_blocks_out_of_range_skipped(oracle)),
    ]
    for name, fn in checks:
        try:
            fn()
        except Exception:  # noqa: BLE001 -- any failure counts as caught
            failed.append(name)
    return failed


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path, golden_dir):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                           "-ffp-contract=off", "-o", str(so), str(path), "-lm"])
    oracle.use_library(str(so))
    try:
        failed = _run_pins(golden_dir)
    finally:
        oracle.use_library(None)
    assert failed, f"mutant {name} passed every pin"


def test_unmutated_oracle_passes_all(golden_dir):
    assert _run_pins(golden_dir) == []
