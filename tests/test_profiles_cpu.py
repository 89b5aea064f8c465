"""The committed ncu evidence is one capture set: every summary under profiles/ names the kernel-source hash
that profiles/traffic.txt is keyed by, and every traffic line parses (path, workload, hash, bytes)."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = os.path.join(ROOT, "profiles")


def _traffic():
    rows = []
    for ln in open(os.path.join(PROFILES, "traffic.txt")):
        if ln.startswith("#") or not ln.strip():
            continue
        f = ln.split()
        assert len(f) == 4, ln
        assert f[0].startswith("path=") and ":M=" in f[1] and re.fullmatch(r"[0-9a-f]{12}", f[2]), ln
        assert int(f[3]) > 0, ln
        rows.append(f)
    return rows


def test_traffic_lines_share_one_source_hash():
    rows = _traffic()
    assert len(rows) >= 6
    assert len({r[2] for r in rows}) == 1


def test_every_summary_names_the_traffic_hash():
    h = _traffic()[0][2]
    summaries = [f for f in os.listdir(PROFILES) if f.endswith(".md")]
    assert summaries
    for f in summaries:
        text = open(os.path.join(PROFILES, f)).read()
        m = re.search(r"Kernel source hash \(bench\.py `kernel_source_hash`, sha256 over `csrc/`\): ([0-9a-f]+)\.", text)
        assert m is not None, f
        assert m.group(1) == h, (f, m.group(1), h)
        assert "--clock-control none" in text, f          # every ncu command leaves the clocks alone
