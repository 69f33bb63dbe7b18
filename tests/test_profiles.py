"""Every ncu command recorded in the committed summaries under profiles/
leaves the GPU clocks alone (--clock-control none).  CPU only."""
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_profile_commands_leave_clocks_alone():
    files = glob.glob(os.path.join(ROOT, "profiles", "*.md")) + glob.glob(os.path.join(ROOT, "profiles", "*.txt"))
    assert files
    for path in files:
        text = open(path).read().replace("\\\n", " ")  # join continued lines
        for cmd in re.findall(r"ncu --[^\n]*", text):
            assert "--clock-control none" in cmd, f"{os.path.basename(path)}: {cmd}"
