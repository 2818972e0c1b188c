"""bench.py's recorded DRAM traffic: used only while a kernel's sources are the ones measured.

The `roofline.traffic` figure comes from `profiles/traffic.json`, keyed on a hash of the files a
kernel is built from.  These checks keep that hash honest: every local header a kernel's source
includes (transitively) is among the hashed files, the kernel is defined in the file named for
it, and a record whose hash differs is not used.
"""
import json
import os
import re

import bench

INCLUDE = re.compile(r'^\s*#\s*include\s+"([^"]+)"', re.M)
ALWAYS = ["kernels.cuh", "ptx.cuh"]  # hashed for every kernel


def _local_includes(name, seen=None):
    seen = set() if seen is None else seen
    path = os.path.join(bench.CSRC, name)
    if name in seen or not os.path.exists(path):
        return seen
    seen.add(name)
    with open(path) as f:
        for inc in INCLUDE.findall(f.read()):
            _local_includes(inc, seen)
    return seen


def test_hashed_files_cover_every_local_include():
    for kernel, files in bench.KERNEL_SOURCES.items():
        hashed = set(files) | set(ALWAYS)
        for f in files:
            assert os.path.exists(os.path.join(bench.CSRC, f)), (kernel, f)
            needed = {n for n in _local_includes(f) if os.path.exists(os.path.join(bench.CSRC, n))}
            assert needed <= hashed, (kernel, sorted(needed - hashed))


def test_each_kernel_is_defined_in_its_first_file():
    for kernel, files in bench.KERNEL_SOURCES.items():
        with open(os.path.join(bench.CSRC, files[0])) as f:
            src = f.read()
        assert re.search(r"__global__[^;{]*\b%s\s*\(" % re.escape(kernel), src), (kernel, files[0])


def test_record_used_only_while_the_hash_matches(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    good = bench.kernel_source_hash("gemm_kernel")
    rec = {"wl_a": {"gemm_kernel": {"dram_bytes_per_launch": 123, "kernel_source_hash": good}},
           "wl_b": {"gemm_kernel": {"dram_bytes_per_launch": 456, "kernel_source_hash": "0" * 16}}}
    (prof / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("wl_a", "gemm_kernel") == 123
    assert bench.recorded_traffic("wl_b", "gemm_kernel") is None
    assert bench.recorded_traffic("wl_c", "gemm_kernel") is None


def test_committed_records_name_their_source_summary():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    for wl, kernels in rec.items():
        for kernel, e in kernels.items():
            assert kernel in bench.KERNEL_SOURCES, (wl, kernel)
            assert e["dram_bytes_per_launch"] > 0
            summaries = re.findall(r"profiles/[\w.\-]+\.md", e["source"])
            assert summaries, (wl, kernel)
            for s in summaries:
                assert os.path.exists(os.path.join(bench.ROOT, s)), s
