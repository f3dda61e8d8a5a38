"""bench.py's host-side helpers (CPU only)."""
import json
import os

import bench


def test_source_digest_ignores_comments_not_code(tmp_path, monkeypatch):
    csrc = tmp_path / "combine_moe_layout_08_b200" / "csrc"
    csrc.mkdir(parents=True)
    src = csrc / "k.cu"
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    src.write_text("// a kernel\n__global__ void k(int* p) { p[0] = 1; }  /* one store */\n")
    d0 = bench.source_digest(["k.cu"])
    src.write_text("// the kernel, reworded\n__global__  void k(int* p) {\n  p[0] = 1;\n}\n")
    assert bench.source_digest(["k.cu"]) == d0
    src.write_text("__global__ void k(int* p) { p[0] = 2; }\n")
    assert bench.source_digest(["k.cu"]) != d0


def test_every_traffic_record_names_existing_sources():
    with open(os.path.join(bench.ROOT, "profiles", "dram_traffic.json")) as f:
        rec = json.load(f)
    for key, r in rec.items():
        kernel, workload = key.split("@")
        assert r["bytes_per_launch"] > 0 and r["sources"]
        assert bench.source_digest(r["sources"])        # files exist and read
        assert os.path.exists(os.path.join(bench.ROOT, r["capture"])), r["capture"]


def test_every_profile_summary_gives_its_command():
    """Each ncu summary under profiles/ states the command that made it: an
    ncu invocation of bench.py (a committed file) with --clock-control none."""
    pdir = os.path.join(bench.ROOT, "profiles")
    names = [n for n in os.listdir(pdir) if n.endswith(".md")]
    assert names
    for n in names:
        text = open(os.path.join(pdir, n)).read()
        assert "ncu " in text and "--clock-control none" in text, n
        assert "python bench.py" in text, n
