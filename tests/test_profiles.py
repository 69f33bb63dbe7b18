"""The committed ncu summaries stay usable by the benchmark: the select
profiles were taken on the current kernel source (else the bench's roofline
traffic reads null), and every recorded ncu command leaves the GPU clocks
alone.  CPU only."""
import glob
import os
import re

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_select_profiles_match_the_kernel_source():
    # c1_vit56: one launch per select (clusters); c4a_long16k: eight launches (phases, global sync)
    c1 = bench.recorded_traffic("c1_vit56", 1, 1)
    c4a = bench.recorded_traffic("c4a_long16k", 3, 8)
    assert c1 is not None and c1 > 0, "profiles/rpc_select_c1_vit56.md predates the select kernel source"
    assert c4a is not None and c4a > 0, "profiles/rpc_select_gs_c4a_long16k.md predates the select kernel source"
    # another launch count is not the same measurement
    assert bench.recorded_traffic("c4a_long16k", 3, 1) is None


def test_profile_commands_leave_clocks_alone():
    files = glob.glob(os.path.join(ROOT, "profiles", "*.md")) + glob.glob(os.path.join(ROOT, "profiles", "*.txt"))
    assert files
    for path in files:
        text = open(path).read()
        for cmd in re.findall(r"ncu --[^\n]*", text):
            assert "--clock-control none" in cmd, f"{os.path.basename(path)}: {cmd}"
