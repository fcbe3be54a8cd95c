"""The committed ncu summaries under profiles/: each names the command that produced it, and the
kernel summaries carry the source hash that bench.py matches before it reports their DRAM
traffic (so a kernel change without a new capture shows here, not as a silently missing
roofline.traffic)."""
import os

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROF = os.path.join(ROOT, "profiles")

KERNEL_SUMMARIES = {
    "decode_megakernel_decode_t1_l48_h2048.txt": bench.DECODE_SOURCES,
    "decode_megakernel_decode_t1_l16_h4096.txt": bench.DECODE_SOURCES,
    "decode_megakernel_decode_t16_l24_h2048.txt": bench.DECODE_SOURCES,
    "prefill_tc_grouped_prefill_t4096_h2048.txt": bench.PREFILL_SOURCES,
}


def test_every_summary_names_its_command_and_is_text():
    names = sorted(os.listdir(PROF))
    assert names, "no profiles"
    for n in names:
        assert n.endswith((".txt", ".md")), n
        text = open(os.path.join(PROF, n)).read()
        assert "ncu " in text and "--clock-control none" in text, n
        assert "bench.py" in text, n
        assert len(text) < 16384, n


@pytest.mark.parametrize("name", sorted(KERNEL_SUMMARIES))
def test_kernel_summary_matches_the_current_sources(name):
    traffic = bench.recorded_traffic(name, KERNEL_SUMMARIES[name])
    assert traffic is not None and traffic > 0, f"{name}: source hash differs from the current kernel sources"
