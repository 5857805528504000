"""Host-side checks of the build script's knob handling and of how bench.py
ties a committed ncu summary to the kernel source it was taken on."""
import json
import os
import subprocess

import bench
from tree_masked_verification_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_build_passes_knobs_as_defines_and_writes_elsewhere(monkeypatch, tmp_path):
    seen = {}

    def fake_run(cmd, check):
        seen["cmd"] = cmd
        out = cmd[cmd.index("-o") + 1]
        open(out, "wb").close()

    monkeypatch.setattr(subprocess, "run", fake_run)
    target = tmp_path / "lib_knobs.so"
    got = build.build(out=str(target), defines=["HTA_KV_STAGES_D128=2", "HTA_EXP2_POLY_EVERY=8"])
    assert got == str(target) and target.exists()
    cmd = seen["cmd"]
    assert "-DHTA_KV_STAGES_D128=2" in cmd and "-DHTA_EXP2_POLY_EVERY=8" in cmd
    assert "arch=compute_100a,code=sm_100a" in cmd
    # every CUDA source of the package goes into the one library
    assert set(build.sources()) <= set(cmd)


def test_committed_prefix_profiles_match_the_kernel_source():
    """Each profiles/prefix_tc_kernel_<workload>.json names the hash of the
    kernel file and its two headers it was captured on; bench.py reports its
    DRAM traffic only while that hash is current."""
    prof_dir = os.path.join(ROOT, "profiles")
    names = [n for n in os.listdir(prof_dir) if n.startswith("prefix_tc_kernel_") and n.endswith(".json")]
    assert names
    sha = bench.prefix_source_sha()
    for n in names:
        with open(os.path.join(prof_dir, n)) as f:
            prof = json.load(f)
        assert prof["source_sha256_16"] == sha, n
        wl = n[len("prefix_tc_kernel_"):-len(".json")]
        assert bench.profiled_traffic(wl) == int(prof["dram_bytes_read"] + prof["dram_bytes_write"])


def test_traffic_is_not_reported_for_another_build(monkeypatch):
    monkeypatch.setenv("LONGSPEC_HTA_LIB", "/nonexistent/lib.so")
    assert bench.profiled_traffic("llama3-8b-32k") is None
