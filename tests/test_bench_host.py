"""Host-side helpers of bench.py, on CPU: the rotating operand sets of the linear timings and the
DRAM-traffic record of the rotation kernel."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_rotating_sets_exceed_twice_the_l2():
    import torch
    a = torch.zeros(1 << 20, dtype=torch.uint8)          # 1 MB
    b = torch.zeros(1 << 18, dtype=torch.float16)        # 0.5 MB
    sets = bench._rotating((a, b))
    per_set = a.numel() + 2 * b.numel()
    assert len(sets) * per_set >= bench.L2_FLUSH_BYTES
    assert (len(sets) - 1) * per_set < bench.L2_FLUSH_BYTES
    assert sets[0][0] is a and sets[0][1] is b           # the first set is the operands themselves
    ptrs = {s[0].data_ptr() for s in sets}
    assert len(ptrs) == len(sets)                         # every other set is its own copy


def test_rotating_sets_keep_a_minimum_for_large_operands():
    import torch
    big = torch.zeros(bench.L2_FLUSH_BYTES // 2 + 1, dtype=torch.uint8)
    assert len(bench._rotating((big,))) == 3


def test_traffic_record_matches_the_rotation_kernel_sources():
    """The committed steady-state traffic record of the rotation kernel applies to the kernel as
    built (its recorded hash covers the kernel's device code); a device-code change without a new
    capture makes the bench report no traffic rather than a stale figure."""
    t = bench.profiled_traffic("rot_quant_llama32_1b")
    assert t is not None and t >= bench.algorithmic_bytes(8192, 2048, 4, 32)
