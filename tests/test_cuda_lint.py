"""Static checks of the CUDA sources, on the CPU.

A warp-synchronous intrinsic whose mask names every lane must be executed by
every lane. Written as the right operand of `&&` or `||`, or as a branch of
`?:`, it is skipped by the lanes the left operand decides; on sm_100a that
raised "an illegal instruction was encountered" once in this library's
history (a vote in the top-k scan). The vote is taken into a variable first.
"""
import glob
import os
import re

CSRC = os.path.join(os.path.dirname(__file__), "..", "logit_kl_divergence_b200", "csrc")
SYNC = r"__(?:all|any|ballot|match_any|match_all|shfl(?:_up|_down|_xor)?|reduce_\w+)_sync\s*\("
SHORT_CIRCUIT = re.compile(r"(?:&&|\|\||\?)\s*!?\s*\(?\s*" + SYNC)


def _code(text):
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return "\n".join(re.sub(r"//.*$", "", ln) for ln in text.splitlines())


def test_no_warp_intrinsic_after_a_short_circuit():
    bad = []
    for path in sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))):
        for n, line in enumerate(_code(open(path, encoding="utf-8").read()).splitlines(), 1):
            if SHORT_CIRCUIT.search(line):
                bad.append(f"{os.path.basename(path)}:{n}: {line.strip()}")
    assert not bad, "warp-synchronous intrinsic on a short-circuited path:\n" + "\n".join(bad)


def test_the_check_catches_the_pattern():
    assert SHORT_CIRCUIT.search("flag = mb >= tf || !__all_sync(0xffffffffu, axl <= kTau);")
    assert SHORT_CIRCUIT.search("x = c ? __shfl_sync(0xffffffffu, v, 0) : 0;")
    assert not SHORT_CIRCUIT.search("const bool direct = !__all_sync(0xffffffffu, axl <= kTau);")
    assert not SHORT_CIRCUIT.search("if (__any_sync(0xffffffffu, a || b)) {")
