"""Source rules the library keeps (read as text, nothing runs): no load with cluster multicast
(the only multicast form is the tcgen05.commit arrive on the CTA pair's barriers), no batched
memcpy entry point, no device trap, and every spin on an mbarrier goes through the bounded
waits of dckv_ptx.cuh."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "learned_kv_cache_dckv_b200", "csrc")


def _sources():
    out = {}
    for d in (CSRC, os.path.join(ROOT, "include"), os.path.join(ROOT, "oracle")):
        for f in sorted(os.listdir(d)):
            if f.endswith((".cu", ".cuh", ".h", ".c", ".cpp")):
                out[os.path.join(d, f)] = open(os.path.join(d, f)).read()
    return out


def test_multicast_only_on_commit_arrives():
    for path, text in _sources().items():
        for line in text.splitlines():
            if "multicast::cluster" in line:
                assert "tcgen05.commit" in line, f"{os.path.basename(path)}: {line.strip()}"


def test_no_batched_memcpy():
    names = ["cuda" + "Memcpy" + k + "Batch" + "Async" for k in ("", "3D")]
    names += ["cu" + "Memcpy" + k + "Batch" + "Async" for k in ("", "3D")]
    for path, text in _sources().items():
        for n in names:
            assert n not in text, os.path.basename(path)


def test_no_device_trap():
    for path, text in _sources().items():
        assert "__trap" not in text and "asm(\"trap" not in text.replace(" ", ""), os.path.basename(path)


def test_mbarrier_spins_are_bounded():
    # every try_wait sits in dckv_ptx.cuh, whose callers loop with a global-timer bound
    for path, text in _sources().items():
        if "try_wait" in text:
            assert os.path.basename(path) == "dckv_ptx.cuh", os.path.basename(path)
    ptx = open(os.path.join(CSRC, "dckv_ptx.cuh")).read()
    for fn in ("mbar_wait", "mbar_drain"):
        body = ptx[ptx.index(f"bool {fn}("):]
        body = body[: body.index("\n}\n")]
        assert "DCKV_WAIT_NS" in body, fn
    assert re.search(r"#define DCKV_WAIT_NS \d+", ptx)
