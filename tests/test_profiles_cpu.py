"""The committed profile records match the sources they describe: the DRAM
traffic and instruction count that bench.py reports for the timed forward kernel
are used only while the kernel's sources hash to the recorded value, so a kernel
edit without a new capture shows up here (and as a null `traffic` in the bench
line)."""
import json
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_traffic_record_matches_kernel_sources():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        ent = json.load(f)["dcnv4_p4_forward"]
    assert ent["kernel_hash"] == bench.kernel_hash()
    assert ent["kernel_sources"] == [os.path.basename(p) for p in bench.KERNEL_SOURCES]
    assert ent["bytes_per_launch"] == ent["dram_bytes_read"] + ent["l2_write_bytes"]
    # the recorded traffic is within 1 % of the algorithmic x + offset + mask + out bytes
    assert abs(ent["bytes_per_launch"] / 37273600 - 1.0) < 0.01
    assert ent["warp_instructions_per_launch"] > 0


def test_profiles_give_their_commands():
    """Every summary gives the command that made it, in a fenced block, running
    committed files only; every ncu command in it leaves the GPU clocks alone."""
    d = os.path.join(ROOT, "profiles")
    for name in os.listdir(d):
        if name.endswith(".md"):
            text = open(os.path.join(d, name), encoding="utf-8").read()
            blocks = text.split("```")[1::2]
            assert blocks and any(("bench.py" in b) or ("python -c" in b) for b in blocks), name
            for b in blocks:
                if "ncu " in b:
                    assert "--clock-control none" in b, name
                assert "_work" not in b, name
