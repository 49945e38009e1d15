"""Host-side rules of the CUDA library that need no GPU, compiled from the
library's own headers with the host C++ compiler.

choose_cluster_size (csrc/cluster_choice.h) picks the cluster size of the fused
decode select: the fewest waves of (batch, kv head) clusters, then the largest
size.  The active-cluster counts below are the ones the occupancy query
reports on a 148-SM B200 at one CTA per SM (15 clusters of 8 or 9 CTAs, 11 of
10, 7 of 12 or 16).  choose_fused_select_size keeps that choice only when all
problems run in one wave (else the library scores in one kernel and selects
in a second)."""
import os
import shutil
import subprocess

import pytest

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "sparse_attention_long_anchor_b200", "csrc")

SIZES = [16, 12, 10, 9, 8]
B200_ACTIVE = [7, 7, 11, 15, 15]

CASES = [
    # (problems, active, fits, expected)
    *[(p, B200_ACTIVE, [1] * 5, 16) for p in range(1, 8)],
    (8, B200_ACTIVE, [1] * 5, 10),      # the Llama-shaped layer: 8 kv heads
    (11, B200_ACTIVE, [1] * 5, 10),
    (12, B200_ACTIVE, [1] * 5, 9),
    (15, B200_ACTIVE, [1] * 5, 9),
    (16, B200_ACTIVE, [1] * 5, 10),     # two waves at 10, 9 or 8: the largest
    (22, B200_ACTIVE, [1] * 5, 10),
    (23, B200_ACTIVE, [1] * 5, 9),
    (64, B200_ACTIVE, [1] * 5, 9),      # batch 8: five waves of 9
    (4, B200_ACTIVE, [0, 1, 1, 1, 1], 12),   # 16-CTA shared memory does not fit
    (4, [0, 0, 11, 15, 15], [1] * 5, 10),     # no large clusters on the device
    (4, B200_ACTIVE, [0, 0, 0, 0, 1], 8),
    (4, [0] * 5, [1] * 5, 0),                 # nothing runs: no fused kernel
    (4, B200_ACTIVE, [0] * 5, 0),
]


def _program() -> str:
    lines = ['#include <cstdio>', '#include "cluster_choice.h"', "int main() {",
             "  const int sizes[5] = {%s};" % ", ".join(map(str, SIZES))]
    for i, (p, act, fits, _) in enumerate(CASES):
        lines.append("  { const int a[5] = {%s}; const bool f[5] = {%s};"
                     % (", ".join(map(str, act)), ", ".join("true" if x else "false" for x in fits)))
        lines.append('    std::printf("%%d\\n", kascade::choose_cluster_size(%dLL, sizes, a, f, 5)); }' % p)
    lines += ["  return 0;", "}"]
    return "\n".join(lines) + "\n"


# (problems, active, fits, expected) for choose_fused_select_size: the same
# choice, kept only when every problem runs in one wave
FUSED_CASES = [
    (1, B200_ACTIVE, [1] * 5, 16),
    (7, B200_ACTIVE, [1] * 5, 16),
    (8, B200_ACTIVE, [1] * 5, 10),      # the Llama-shaped layer at batch 1: fused
    (15, B200_ACTIVE, [1] * 5, 9),      # 15 clusters of 9 run at once
    (16, B200_ACTIVE, [1] * 5, 0),      # two waves: scoring kernel + select
    (64, B200_ACTIVE, [1] * 5, 0),      # batch 8: five waves
    (4, B200_ACTIVE, [0, 0, 0, 0, 1], 8),
    (16, B200_ACTIVE, [0, 0, 0, 0, 1], 0),
    (4, [0] * 5, [1] * 5, 0),
]


def _compile_and_run(tmp_path_factory, body):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    d = tmp_path_factory.mktemp("host_rules")
    src, exe = d / "t.cpp", d / "t"
    src.write_text(body)
    subprocess.run([cxx, "-std=c++17", "-O1", "-I", CSRC, str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    return [int(x) for x in out]


def _fused_program() -> str:
    lines = ['#include <cstdio>', '#include "cluster_choice.h"', "int main() {",
             "  const int sizes[5] = {%s};" % ", ".join(map(str, SIZES))]
    for p, act, fits, _ in FUSED_CASES:
        lines.append("  { const int a[5] = {%s}; const bool f[5] = {%s};"
                     % (", ".join(map(str, act)), ", ".join("true" if x else "false" for x in fits)))
        lines.append('    std::printf("%%d\\n", kascade::choose_fused_select_size(%dLL, sizes, a, f, 5)); }' % p)
    lines += ["  return 0;", "}"]
    return "\n".join(lines) + "\n"


@pytest.fixture(scope="module")
def fused_chosen(tmp_path_factory):
    return _compile_and_run(tmp_path_factory, _fused_program())


@pytest.mark.parametrize("case", range(len(FUSED_CASES)))
def test_fused_select_one_wave_rule(fused_chosen, case):
    problems, active, fits, expected = FUSED_CASES[case]
    assert fused_chosen[case] == expected, (problems, active, fits)


# choose_overlap_cluster_size over the short-list decode's sizes: the largest
# size at which twice the problems are resident, else the largest with one
# wave, else 0 (the bulk mode)
SIZES0 = [16, 15, 14, 13, 12, 10, 8, 4]
ACT0 = [14, 15, 17, 18, 21, 22, 33, 71]          # a plausible two-CTAs-per-SM device
FIT_LLAMA = [1, 1, 1, 1, 0, 0, 0, 0]             # 3277 keys: 256 per CTA or fewer needs 13 CTAs or more
OVERLAP_CASES = [
    (8, ACT0, FIT_LLAMA, 14),      # 14 and 15 < 16: 14 CTAs (17 clusters resident)
    (8, [14, 16, 17, 18, 21, 22, 33, 71], FIT_LLAMA, 15),
    (7, ACT0, FIT_LLAMA, 16),      # 14 >= 2 x 7
    (2, ACT0, [1] * 8, 16),
    (16, ACT0, FIT_LLAMA, 14),     # nothing holds 32: the largest size with one wave
    (40, ACT0, [1] * 8, 4),        # 71 < 80: one wave only at 4
    (64, ACT0, FIT_LLAMA, 0),      # batch 8 of the Llama layer: no one-wave size, the bulk mode runs
    (8, ACT0, [0] * 8, 0),         # no size keeps the short-list mode: the bulk mode runs
]


def _overlap_program() -> str:
    lines = ['#include <cstdio>', '#include "cluster_choice.h"', "int main() {",
             "  const int sizes[8] = {%s};" % ", ".join(map(str, SIZES0))]
    for p, act, fits, _ in OVERLAP_CASES:
        lines.append("  { const int a[8] = {%s}; const bool f[8] = {%s};"
                     % (", ".join(map(str, act)), ", ".join("true" if x else "false" for x in fits)))
        lines.append('    std::printf("%%d\\n", kascade::choose_overlap_cluster_size(%dLL, sizes, a, f, 8)); }' % p)
    lines += ["  return 0;", "}"]
    return "\n".join(lines) + "\n"


@pytest.fixture(scope="module")
def overlap_chosen(tmp_path_factory):
    return _compile_and_run(tmp_path_factory, _overlap_program())


@pytest.mark.parametrize("case", range(len(OVERLAP_CASES)))
def test_decode_overlap_rule(overlap_chosen, case):
    problems, active, fits, expected = OVERLAP_CASES[case]
    assert overlap_chosen[case] == expected, (problems, active, fits)


@pytest.fixture(scope="module")
def chosen(tmp_path_factory):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    d = tmp_path_factory.mktemp("host_rules")
    src, exe = d / "t.cpp", d / "t"
    src.write_text(_program())
    subprocess.run([cxx, "-std=c++17", "-O1", "-I", CSRC, str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    return [int(x) for x in out]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_cluster_size_rule(chosen, case):
    problems, active, fits, expected = CASES[case]
    assert chosen[case] == expected, (problems, active, fits)


def test_rule_never_picks_a_size_that_cannot_run(chosen):
    for (problems, active, fits, _), got in zip(CASES, chosen):
        if got:
            i = SIZES.index(got)
            assert active[i] > 0 and fits[i]
