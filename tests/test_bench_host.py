"""Host-side pieces of bench.py that need no GPU: the DRAM traffic it reports
for the dominant kernel comes from a committed ncu summary only while that
summary was taken on the kernel's current source."""
import re
import sys
from pathlib import Path

ROOT = Path(__file__).resolve().parents[1]
sys.path.insert(0, str(ROOT))

import bench  # noqa: E402


def test_profile_traffic_is_gated_on_the_source_hash(tmp_path):
    md = (ROOT / "profiles" / "skinny_w8a8_decode.md").read_text()
    traffic = float(re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", md).group(1))
    src = ROOT / "moe_hadamard128_act_b200" / "csrc" / "k_skinny.cu"
    got = bench.kernel_traffic("skinny_w8a8_decode", src)
    assert got is None or got == traffic  # the number itself, or nothing once the source has moved on
    edited = tmp_path / "k_skinny.cu"
    edited.write_bytes(src.read_bytes() + b"\n// edited\n")
    assert bench.kernel_traffic("skinny_w8a8_decode", edited) is None
    assert bench.kernel_traffic("no_such_profile", src) is None


def test_every_profile_names_its_command_and_source():
    for md in sorted((ROOT / "profiles").glob("*.md")):
        text = md.read_text()
        assert "ncu " in text and "--clock-control none" in text, md.name
        assert re.search(r"source_sha256[^:]*:\s*[0-9a-f]{64}", text), md.name
