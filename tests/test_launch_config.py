"""The launch configuration bench.py times for each named decode workload
(host logic only, no GPU): the step and split-KV partition of each, so that
the benchmarked configuration cannot drift from the one the workload names
and the full-size parity tests check."""

import re

import pytest

import workload
from paged_kv_cache_369_b200.runner import default_mode, default_partition_size


def test_long_context_keeps_its_prescribed_partitions():
    """The long-context E4M3 workload names split-KV partitions of 512
    tokens; the default step uses exactly that size."""
    m = re.search(r"split (\d+)", workload.gen.CONFIG_NAMES[4])
    assert m, workload.gen.CONFIG_NAMES[4]
    assert default_partition_size(None, 4) == int(m.group(1)) == 512


@pytest.mark.parametrize("cfg,P,mode", [(1, 1024, "fused"), (2, 1024, "fused"), (3, 1024, "fused_single"),
                                        (4, 512, "fused"), (5, 768, "fused")])
def test_default_step_per_workload(cfg, P, mode):
    assert default_partition_size(None, cfg) == P
    assert default_mode(cfg) == mode


def test_partitions_are_whole_tiles():
    """Every default partition is a positive multiple of 16 tokens (the
    C ABI rejects anything else)."""
    for cfg in range(1, 6):
        P = default_partition_size(None, cfg)
        assert P > 0 and P % 16 == 0
