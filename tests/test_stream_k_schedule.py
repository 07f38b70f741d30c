"""CPU check of the CTA-pair GEMM's work lists and tile plan.

Builds tests/sk_schedule_check.cpp against the library's own schedule code
(int8_mixed_precision_rowwise_b200/csrc/sched.h) with g++ and runs it over the
five workloads' prefill shapes and a few thousand seeded random ones: every
(tile, K stage) processed once, at most one parked part per pair and first in
its stream-K range, every fix-up last and matched by the previous pair's park.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "int8_mixed_precision_rowwise_b200", "csrc")
SRC = os.path.join(ROOT, "tests", "sk_schedule_check.cpp")


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("no g++")
    exe = str(tmp_path_factory.mktemp("sk") / "sk_schedule_check")
    subprocess.run([gxx, "-std=c++17", "-O1", "-Wall", "-Werror", "-I", CSRC, "-o", exe, SRC], check=True)

    def run(shapes):
        inp = "".join(f"{M} {N} {K} {P}\n" for M, N, K, P in shapes)
        r = subprocess.run([exe], input=inp, capture_output=True, text=True)
        assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
        return [tuple(int(v) for v in line.split()[:7]) for line in r.stdout.splitlines()]
    return run


def test_bloom_and_prefill_plans(checker):
    """On 74 pairs (a 148-SM B200) the four BLOOM linears at 2048 tokens run
    256-wide tiles with their last 86 / 78 / 90 / 78 tiles stream-K; the
    2048 x 16384 x 4096 prefill keeps whole tiles (512 tiles fill 6.9 rounds)."""
    out = checker([(2048, 43008, 14336, 74), (2048, 14336, 14336, 74), (2048, 57344, 14336, 74),
                   (2048, 14336, 57344, 74), (2048, 16384, 4096, 74)])
    assert [o[4:] for o in out] == [(256, 1, 86), (256, 1, 78), (256, 1, 90), (256, 1, 78), (256, 0, 0)]


def test_random_shapes(checker):
    rng = np.random.default_rng(7)
    shapes = []
    for _ in range(3000):
        M = int(rng.integers(256, 6000))
        N = int(rng.integers(1, 4500)) * 16
        K = int(rng.integers(1, 600)) * 16
        P = int(rng.choice([74, 66, 80, 10, 1]))
        shapes.append((M, N, K, P))
    out = checker(shapes)
    assert len(out) == len(shapes)
    assert sum(o[5] for o in out) > 500  # a good share of them exercise stream-K
