"""bench.py reports the attention kernel's DRAM traffic only from a committed
capture of the same kernel source: every entry of its traffic table names a
source hash and a figure that the capture summary under profiles/ records,
and a source that no capture covers gets null."""
import importlib.util
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILE = os.path.join(ROOT, "profiles", "attn_fwd_kernel_dram_ring_workloads.md")


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_traffic_entries_are_backed_by_the_capture_summary():
    b = _bench()
    text = open(PROFILE).read()
    assert b.ATTN_TRAFFIC, "no traffic entries"
    for (src_hash, workload), value in b.ATTN_TRAFFIC.items():
        assert re.fullmatch(r"[0-9a-f]{16}", src_hash)
        assert src_hash in text, f"capture summary does not name source {src_hash}"
        row = next(line for line in text.splitlines() if line.startswith(f"| `{workload}`"))
        # the table's traffic column (GB), to the summary's rounding
        traffic_gb = float(row.split("|")[5].split()[0])
        assert abs(value / 1e9 - traffic_gb) <= 0.0015, (workload, value, traffic_gb)


def test_source_without_a_capture_reports_null():
    b = _bench()
    assert b.ATTN_TRAFFIC.get(("0" * 16, "varlen_zigzag_128k")) is None
    current = b.attn_src_hash()
    assert re.fullmatch(r"[0-9a-f]{16}", current)
    covered = {h for h, _ in b.ATTN_TRAFFIC}
    if current not in covered:
        assert all(b.ATTN_TRAFFIC.get((current, w)) is None for _, w in b.ATTN_TRAFFIC)
