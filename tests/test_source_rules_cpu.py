"""Static rules of the CUDA sources, checked on the text (no device):

* every wait is bounded: the raw mbarrier wait and the global-flag poll exist
  only inside the bounded helpers of csrc/tc.cuh (`mbar_wait`,
  `spin_until_geq`), which give up after a time limit, set the device
  status word and return -- so no kernel can spin forever;
* no kernel stops the device on purpose: no `__trap`, no device `assert`;
* no bulk or tensor copy multicasts across a cluster;
* every MMA, scale-factor copy and commit is issued from one lane.
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


_ONE_LANE = (r"if\s*\(\s*elect_one\(\)\s*\)", r"if\s*\(\s*leader\s*\)", r"if\s*\(\s*lane\s*==\s*0\s*\)")
_TENSOR_ISSUE = re.compile(r"\b(mma_f16|mma_f16_ta|mma_nvf4|tc_cp_32x128b_x4|tc_commit)\s*\(")


def _single_lane_violations(code):
    """Calls that issue tensor-core work (MMA, scale-factor copy, commit)
    outside a block or statement guarded to one lane of the warp."""
    bad = []
    stack = []  # the statement text that opened each enclosing brace
    stmt = ""
    i = 0
    while i < len(code):
        ch = code[i]
        m = _TENSOR_ISSUE.match(code, i) if (i == 0 or not (code[i - 1].isalnum() or code[i - 1] == "_")) else None
        if m:
            guarded = any(re.search(p, s) for p in _ONE_LANE for s in stack + [stmt])
            if not guarded:
                bad.append(code[max(0, i - 60):i + 40].replace("\n", " "))
            stmt += m.group(0)
            i = m.end()
            continue
        if ch == "{":
            stack.append(stmt)
            stmt = ""
        elif ch == "}":
            if stack:
                stack.pop()
            stmt = ""
        elif ch == ";":
            stmt = ""
        else:
            stmt += ch
        i += 1
    return bad


def test_tensor_instructions_issue_from_one_lane():
    # tc.cuh defines the wrappers; every kernel that calls them issues each
    # MMA, scale-factor copy and commit from a single lane (elected, or lane
    # 0), so that the commit tracks the MMAs of the same thread and no warp
    # issues a product 32 times
    for name, text in _sources():
        if name == "tc.cuh":
            continue
        bad = _single_lane_violations(_code(text))
        assert not bad, f"{name}: tensor instructions outside a one-lane guard: {bad[:3]}"


def test_single_lane_rule_catches_an_unguarded_issue():
    assert _single_lane_violations("void f() { if (leader) { mma_f16(a, b); tc_commit(x); } }") == []
    assert _single_lane_violations("void f() { if (elect_one()) tc_commit(x); }") == []
    assert _single_lane_violations("void f() { for (;;) { mma_nvf4(a); } }")
    assert _single_lane_violations("void f() { if (leader) { x(); } tc_commit(y); }")
