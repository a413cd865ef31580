"""The committed measurement evidence is self-consistent: every DRAM-traffic
record names an ncu summary that exists, and every summary gives the command
that produced it (with the clock control left alone)."""
import json
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = os.path.join(ROOT, "profiles")


def test_traffic_records_cite_existing_summaries():
    with open(os.path.join(PROFILES, "traffic.json")) as f:
        records = json.load(f)
    assert records
    for key, rec in records.items():
        assert rec["dram_bytes_per_launch"] > 0, key
        for name in re.findall(r"profiles/([\w.\-]+\.md)", rec["how"]):
            assert os.path.exists(os.path.join(PROFILES, name)), (key, name)


def test_summaries_give_their_command():
    for name in os.listdir(PROFILES):
        if not name.endswith(".md"):
            continue
        text = open(os.path.join(PROFILES, name)).read()
        assert "ncu " in text, name
        assert "--clock-control none" in text, name
