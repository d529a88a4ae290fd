"""Source checks (CPU): constructs the library must never contain.

* no TMA or bulk load with cluster multicast in any CUDA source (every CTA loads its own tiles);
* no batched-memcpy runtime or driver API anywhere in the code (one cudaMemcpyAsync per copy);
* no device trap: kernels report failures through the status word and return;
* every mbarrier wait goes through the bounded helpers of ptx.cuh (no raw wait elsewhere);
* every ncu command recorded under profiles/ leaves the GPU clocks alone;
* nothing changes GPU clocks or other persistent GPU settings.
"""
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = sorted(glob.glob(os.path.join(ROOT, "fwd_bwd_b200", "csrc", "*.cu*")) +
              glob.glob(os.path.join(ROOT, "include", "*.h")))
CODE = CUDA + sorted(glob.glob(os.path.join(ROOT, "fwd_bwd_b200", "*.py")) +
                     glob.glob(os.path.join(ROOT, "tests", "*.py")) +
                     glob.glob(os.path.join(ROOT, "oracle", "*.py")) +
                     [os.path.join(ROOT, "bench.py"), os.path.join(ROOT, "__graft_entry__.py")])


def _read(path):
    return open(path, encoding="utf-8").read()


def _strip_comments(src):
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return re.sub(r"//[^\n]*", "", src)


def test_sources_found():
    assert len(CUDA) >= 8 and len(CODE) >= 30


def test_no_cluster_multicast_loads():
    qualifier = "multicast" + "::" + "cluster"  # spelled apart so this file names no such load
    for path in CUDA:
        assert qualifier not in _read(path), path


def test_no_batched_memcpy():
    names = ["Memcpy" + "Batch", "Memcpy3D" + "Batch"]  # spelled apart on purpose
    for path in CODE:
        src = _read(path)
        for n in names:
            assert n not in src, (path, n)


def test_no_device_trap():
    for path in CUDA:
        src = _strip_comments(_read(path))
        assert "__trap" not in src and not re.search(r"\btrap\s*;", src), path
        assert not re.search(r"\bassert\s*\(", src), path


def test_mbarrier_waits_are_bounded():
    for path in CUDA:
        if os.path.basename(path) == "ptx.cuh":
            continue
        src = _strip_comments(_read(path))
        assert "mbarrier.try_wait" not in src and "mbarrier.wait" not in src, path
    ptx = _strip_comments(_read(os.path.join(ROOT, "fwd_bwd_b200", "csrc", "ptx.cuh")))
    # the one raw wait loop is bounded by a global-timer limit and records a timeout
    assert "record_timeout(site)" in ptx and "limit_ns" in ptx


def test_profile_commands_leave_clocks_alone():
    seen = 0
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        text = _read(path)
        # an ncu command may continue over backslash-newlines
        for cmd in re.findall(r"^ncu .*?(?<!\\)$", text, flags=re.M | re.S):
            seen += 1
            assert "--clock-control none" in cmd, (path, cmd[:80])
    assert seen >= 5


def test_no_gpu_setting_changes():
    # (cudaDeviceReset is allowed: it ends only the calling process's own context)
    bad = [r"nvidia-smi[^\n]*\s-(lgc|ac|pm|rgc|rac|mig|c|e|pl)\b", r"nvmlDeviceSet"]
    for path in CODE:
        src = _read(path)
        if os.path.basename(path) == "test_source_rules.py":
            continue
        for pat in bad:
            assert not re.search(pat, src), (path, pat)
