"""The committed ncu evidence is usable as it stands: every summary under
profiles/ is short text naming the full command that made it (ncu with
--clock-control none, running committed files only), and every DRAM-traffic
entry the bench reads points at such a summary and carries the source hash
that decides whether the bench may still quote it."""
import json
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROF = os.path.join(ROOT, "profiles")


def _summaries():
    return sorted(f for f in os.listdir(PROF) if f.endswith(".md"))


def test_profiles_holds_short_text_only():
    for f in os.listdir(PROF):
        assert os.path.splitext(f)[1] in (".md", ".txt", ".json"), f"{f}: raw or binary output belongs elsewhere"
        assert os.path.getsize(os.path.join(PROF, f)) < 64 * 1024, f"{f} is not a short summary"


def test_every_summary_names_its_ncu_command():
    assert _summaries()
    for f in _summaries():
        text = open(os.path.join(PROF, f)).read()
        cmds = [ln for ln in text.splitlines() if re.match(r"\s*ncu\s", ln)]
        assert cmds, f"{f}: no ncu command line"
        for c in cmds:
            assert "--clock-control none" in c, f"{f}: ncu without --clock-control none"
            assert "python bench.py" in c, f"{f}: the command should run the committed bench"
            assert "_work" not in c, f"{f}: the command runs a scratch file"


def test_traffic_entries_point_at_committed_summaries():
    d = json.load(open(os.path.join(PROF, "traffic.json")))
    entries = {k: v for k, v in d.items() if not k.startswith("_")}
    assert entries
    for key, e in entries.items():
        assert re.fullmatch(r"[0-9a-f]{16}", e["source_sha"]), key
        assert e["dram_bytes_per_launch_full_size"] > 0, key
        assert os.path.exists(os.path.join(ROOT, e["profile"])), f"{key}: {e['profile']} is missing"
        kernel, workload, proj = key.split(":")
        assert proj in ("gate_up", "down"), key
