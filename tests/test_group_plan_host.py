"""CPU test of the wide group-128 kernel's work-unit schedule.

The kernel takes its units from csrc/group_plan.h; this test compiles the
same header into a small host program (tests/group_plan_check.cpp) and
checks the schedule for many tile counts, group counts and SM counts: every
(tile, group) computed exactly once, a cut tile's first part on another CTA
and finished before its second part starts (counting tile-times per CTA),
and the longest CTA at (T - r) / P + 1/2 tile-times when the last wave is
cut, never above the whole-tile schedule."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "w8a8_int8_quantized_qk_b200", "csrc")


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no C++ compiler")
    exe = str(tmp_path_factory.mktemp("plan") / "group_plan_check")
    subprocess.run([cxx, "-O1", "-std=c++17", "-Wall", "-Werror", "-I", CSRC, "-o", exe,
                    os.path.join(ROOT, "tests", "group_plan_check.cpp")], check=True)
    return exe


def _run(exe, tiles, groups, sms):
    r = subprocess.run([exe, str(tiles), str(groups), str(sms)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    _, cut, longest = r.stdout.split()
    return int(cut), float(longest)


def test_group128_workload_cuts_the_last_wave(checker):
    # 2048 x 8192 in 128 x 256 tiles = 512 tiles, 64 groups, 148 SMs:
    # 68 tail tiles cut, 3.5 tile-times instead of 4
    cut, longest = _run(checker, 512, 64, 148)
    assert cut == 68 and longest == pytest.approx(3.5)


def test_group128_workload_on_pairs_cuts_the_last_wave(checker):
    # the CTA-pair kernel: 2048 x 8192 in 256 x 256 tiles = 256 tiles, 64
    # groups, 74 pairs: 34 tail tiles cut, 3.5 tile-times instead of 4
    cut, longest = _run(checker, 256, 64, 74)
    assert cut == 34 and longest == pytest.approx(3.5)


@pytest.mark.parametrize("sms", [1, 2, 3, 7, 74, 132, 148])
@pytest.mark.parametrize("groups", [1, 2, 3, 17, 64])
def test_schedule_invariants(checker, sms, groups):
    for tiles in list(range(1, 3 * sms + 4)) + [5 * sms + sms // 2, 9 * sms + 1]:
        cut, longest = _run(checker, tiles, groups, sms)
        if groups < 2 or tiles <= sms:
            assert cut == 0
        if cut == 0:
            assert longest == pytest.approx(-(-tiles // min(tiles, sms)))
