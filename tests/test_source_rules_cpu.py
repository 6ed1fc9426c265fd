"""Static rules of the CUDA sources, checked on the text (no device):

* every wait is bounded: the raw mbarrier wait and the global-flag poll exist
  only inside the bounded helpers of csrc/tc.cuh (`mbar_wait`,
  `spin_until_geq`), which give up after a time limit, set the device
  status word and return -- so no kernel can spin forever;
* no kernel stops the device on purpose: no `__trap`, no device `assert`;
* no bulk or tensor copy multicasts across a cluster.
"""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bit_quantization_b200", "csrc")


def _sources():
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(CSRC, name)) as f:
                yield name, f.read()


def _code(text):
    """The text without // comments (string literals of inline PTX stay)."""
    return "\n".join(line.split("//", 1)[0] for line in text.splitlines())


def test_raw_waits_only_inside_the_bounded_helpers():
    for name, text in _sources():
        code = _code(text)
        for pat in (r"mbarrier\.try_wait", r"mbarrier\.test_wait", r"ld\.acquire"):
            if name == "tc.cuh":
                continue
            assert not re.search(pat, code), f"{name}: raw {pat} outside csrc/tc.cuh"
        if name != "tc.cuh":
            assert "mbar_try_wait(" not in code, f"{name}: unbounded single-try wait used directly"


def test_bounded_helpers_have_a_time_limit():
    text = _code(dict(_sources())["tc.cuh"])
    for helper in ("mbar_wait", "spin_until_geq"):
        m = re.search(r"\b" + helper + r"\([^)]*\)\s*\{(.*?)\n\}", text, re.S)
        assert m, f"{helper} not found"
        body = m.group(1)
        assert "globaltimer" in body, f"{helper}: no time limit"
        assert "set_device_status" in body, f"{helper}: gives up without recording it"


def test_no_deliberate_device_stops():
    for name, text in _sources():
        code = _code(text)
        assert "__trap" not in code, name
        assert not re.search(r"(?<![_\w])assert\s*\(", code), f"{name}: device assert"


def test_no_cluster_multicast_copies():
    for name, text in _sources():
        assert "multicast::cluster" not in _code(text), name
