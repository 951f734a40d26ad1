"""The build fingerprints do not depend on where the repository is checked out: a GPU
box runs the same tree from a scratch path, and the library stamp and the profiler
counters keyed to a kernel's sources must be recognised there."""
import importlib.util
import json
import os
import shutil

from block_scaled_fp4_04_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_build_copy(tmp_path):
    repo = tmp_path / "elsewhere" / "repo"
    pkg = repo / "block_scaled_fp4_04_b200"
    shutil.copytree(os.path.join(ROOT, "block_scaled_fp4_04_b200", "csrc"), pkg / "csrc")
    shutil.copy(os.path.join(ROOT, "block_scaled_fp4_04_b200", "build.py"), pkg / "build.py")
    shutil.copytree(os.path.join(ROOT, "include"), repo / "include")
    spec = importlib.util.spec_from_file_location("relocated_build", pkg / "build.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_flags_leave_out_the_checkout_location():
    assert ROOT not in build._flags_id()


def test_fingerprints_are_the_same_from_another_directory(tmp_path):
    moved = _load_build_copy(tmp_path)
    assert moved.ROOT != build.ROOT
    assert moved._fingerprint() == build._fingerprint()
    srcs = ["csrc/fp4_decode.cu", "csrc/fp4_ptx.cuh"]
    assert moved.sources_fingerprint(srcs) == build.sources_fingerprint(srcs)


def test_traffic_entries_name_existing_sources():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        entries = json.load(f)
    for key, e in entries.items():
        for rel in e.get("sources", []):
            assert os.path.exists(os.path.join(ROOT, "block_scaled_fp4_04_b200", rel)), (key, rel)
