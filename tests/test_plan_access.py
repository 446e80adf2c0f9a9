"""Host replay of every kernel memory access against the library's plan (CPU).

plan_access_check.cpp includes the library's planner and walks the kernels'
loops with their index arithmetic; see its header for what is checked.
"""
import os
import subprocess
import tempfile

import pytest

from wtconv_inputs import NAMED, sweep_cases

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "plan_access_check.cpp")

EDGE = [
    (3, 5, 56, 56, 5, 3, 0), (1, 1, 8, 8, 5, 3, 0), (1, 1, 16, 16, 7, 4, 0), (2, 3, 24, 40, 3, 3, 0),
    (1, 2, 32, 32, 3, 4, 0), (1, 2, 64, 64, 5, 4, 0), (1, 2, 12, 8, 1, 0, 0), (1, 2, 4, 4, 7, 2, 0),
    (2, 2, 8, 4, 3, 2, 1), (1, 1, 64, 4, 7, 2, 0), (5, 3, 20, 12, 5, 2, 1), (1, 1, 2, 4, 3, 1, 0),
    (1, 1, 64, 64, 7, 6, 0), (1, 1, 4, 4, 1, 1, 1),
    # not multiples of 2^L (zero-padded on chip), incl. strips
    (2, 3, 13, 12, 5, 2, 0), (2, 3, 20, 16, 3, 3, 0), (1, 2, 9, 8, 7, 4, 0), (2, 3, 17, 8, 3, 1, 0),
    (2, 3, 13, 16, 5, 2, 1), (1, 1, 250, 248, 5, 4, 0), (3, 2, 30, 28, 5, 3, 0), (1, 1, 100, 40, 5, 3, 1),
    # deepest levels, bf16 with k = 7, one channel over many batch elements, padded L = 6
    (1, 2, 32, 32, 3, 5, 0), (2, 2, 24, 24, 7, 3, 1), (130, 1, 16, 16, 5, 2, 0), (1, 2, 40, 36, 5, 6, 0),
    (2, 1, 60, 64, 3, 6, 0), (1, 1, 70, 68, 5, 6, 0),
    # clusters of 4 and 16 strips at the sweep's channel counts and batch rule
    (14, 128, 192, 192, 5, 1, 0), (7, 256, 192, 192, 3, 4, 0), (28, 64, 192, 192, 7, 1, 1),
    (10, 64, 320, 320, 3, 1, 0), (1, 512, 320, 320, 5, 1, 1),
    # strips without the pyramid (L = 0) and with levels past it (L = 5, 6): halo rows sent after
    # the analysis instead of from inside it
    (1, 2, 256, 256, 5, 0, 0), (1, 2, 256, 256, 3, 0, 1), (1, 1, 256, 256, 5, 5, 0), (1, 1, 512, 64, 5, 6, 0),
]


@pytest.fixture(scope="module")
def checker():
    d = tempfile.mkdtemp()
    exe = os.path.join(d, "plan_access_check")
    subprocess.run(["g++", "-O2", "-std=c++17", "-o", exe, SRC], check=True, capture_output=True)
    return exe


def _cases():
    out = [(c.B, c.C, c.H, c.W, c.k, c.L, 1 if c.dtype == "bf16" else 0) for c in NAMED.values()]
    out += EDGE
    seen = set()
    for c in sweep_cases():  # the sweep's distinct plane geometries (B and C do not change the plan)
        key = (c.H, c.W, c.k, c.L)
        if key not in seen:
            seen.add(key)
            out.append((2, 3, c.H, c.W, c.k, c.L, 0))
    return out


@pytest.mark.parametrize("case", _cases(), ids=lambda c: "x".join(map(str, c)))
def test_every_access_in_bounds(checker, case):
    r = subprocess.run([checker, *map(str, case)], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip().endswith("OK"), r.stdout + r.stderr


# NHWC activations (layout 1): element-by-element staging and stores; the
# checker also verifies that the kernels' NHWC element map covers the tensor
# exactly once.  Includes shapes whose rows are not whole 16-byte chunks
# (allowed in NHWC only), strips and padded planes.
NHWC = [
    (3, 5, 56, 56, 5, 3, 0), (2, 4, 56, 56, 5, 3, 1), (2, 3, 13, 12, 5, 2, 1), (1, 2, 12, 8, 1, 0, 0),
    (2, 3, 24, 40, 3, 3, 1), (1, 2, 128, 128, 5, 2, 0), (1, 1, 250, 248, 5, 4, 1), (3, 2, 30, 28, 5, 3, 0),
    (2, 2, 64, 64, 7, 4, 0), (5, 3, 20, 12, 5, 2, 1),
    # channel octets (C a multiple of 8, whole planes of a multiple of 32 pixels)
    (3, 16, 56, 56, 5, 3, 0), (2, 8, 32, 32, 3, 2, 1), (2, 16, 56, 56, 7, 0, 0), (5, 8, 16, 16, 1, 2, 1),
    (1, 24, 64, 64, 5, 4, 0), (2, 8, 8, 8, 5, 1, 0), (32, 96, 56, 56, 5, 3, 0), (64, 96, 56, 56, 5, 3, 1),
    # runs of an even number of pixels that is not a multiple of 4 (two pixels a step)
    (3, 16, 28, 28, 5, 2, 0), (2, 8, 28, 28, 3, 2, 1), (32, 192, 28, 28, 5, 2, 0), (2, 8, 28, 28, 7, 0, 0),
    (2, 8, 12, 12, 3, 1, 1), (5, 8, 20, 12, 3, 1, 0),
    # levels past the pyramid
    (2, 8, 64, 64, 3, 5, 0), (2, 16, 32, 32, 5, 5, 1),
]


@pytest.mark.parametrize("case", NHWC, ids=lambda c: "x".join(map(str, c)) + "_nhwc")
def test_every_access_in_bounds_nhwc(checker, case):
    r = subprocess.run([checker, *map(str, case), "1"], capture_output=True, text=True)
    assert r.returncode == 0 and r.stdout.strip().endswith("OK") and "each addressed once" in r.stdout, \
        r.stdout + r.stderr
    # Channel octets exactly where C is a multiple of 8 on whole planes of a multiple of 16 pixels
    # (every case here fits the octet buffer).
    B, C, H, W, k, L, _ = case
    m = 1 << L
    whole = H % m == 0 and W % m == 0 and H * W <= 64 * 64
    octets = C % 8 == 0 and whole and (H * W) % 16 == 0
    fused = [l for l in r.stdout.splitlines() if l.startswith("fused(kind")]
    assert len(fused) == 2 and all(("channel octets" in l) == octets for l in fused), r.stdout
    # The weight gradient takes octets only where it still runs two CTAs an SM (the stage-1 planes).
    bwdw = next(l for l in r.stdout.splitlines() if l.startswith("bwdw:"))
    assert ("channel octets" in bwdw) == (octets and (H, W) != (64, 64)), bwdw


@pytest.mark.parametrize("case,strips,alias", [
    ((1, 1, 256, 256, 5, 4, 0), 8, True),    # DY would not fit beside two staged strips at 8 strips
    ((2, 2, 128, 128, 5, 4, 0), 2, True),
    ((2, 2, 128, 128, 5, 3, 0), 2, False),   # fits with its own DY buffer
    ((3, 5, 56, 56, 5, 3, 0), 1, False),     # whole planes never alias
])
def test_weight_gradient_strip_choice(checker, case, strips, alias):
    # The fewest strips that fit; dy read from its staging only when that is what makes them fit.
    out = subprocess.run([checker, *map(str, case)], capture_output=True, text=True).stdout
    line = next(l for l in out.splitlines() if l.startswith("bwdw:"))
    assert f"strips {strips}" in line, line
    assert ("dy read from staging" in line) == alias, line


@pytest.mark.parametrize("case,one_pass", [
    # Measured on B200 (the shape sweep and the stage shapes): the one pass is
    # faster at 32x32, L = 1 and at 64x64, L >= 3, slower elsewhere.
    ((4, 64, 32, 32, 5, 1, 0), True), ((4, 64, 32, 32, 3, 1, 0), True),
    ((4, 64, 64, 64, 5, 3, 0), True), ((4, 64, 64, 64, 5, 4, 0), True), ((4, 64, 64, 64, 3, 4, 0), True),
    ((4, 64, 32, 32, 5, 2, 0), False), ((4, 64, 32, 32, 5, 3, 0), False), ((4, 64, 64, 64, 5, 1, 0), False),
    ((4, 64, 64, 64, 3, 2, 0), False),
    ((32, 96, 56, 56, 5, 3, 0), False), ((32, 192, 28, 28, 5, 2, 0), False), ((64, 96, 56, 56, 5, 3, 1), False),
    # NHWC (8th field 1): where both passes gather element by element the one pass (measured
    # 1.2-1.45x faster at these six shapes); where the one pass runs on channel octets, the one pass
    # (0.51-1.01x the two passes at eleven shapes, stage1 252 vs 274 us); 28x28 planes (two pixels
    # a step) keep the one pass off octets and the rule above (stage2: two passes, 143.5 vs 149.5 us)
    ((32, 100, 56, 56, 5, 3, 0, 1), True), ((256, 12, 32, 32, 3, 1, 0, 1), True), ((64, 20, 28, 28, 5, 2, 0, 1), True),
    ((128, 36, 32, 32, 5, 4, 0, 1), True), ((16, 60, 64, 64, 3, 2, 0, 1), True), ((512, 6, 16, 16, 3, 2, 0, 1), True),
    ((32, 96, 56, 56, 5, 3, 0, 1), True), ((64, 96, 56, 56, 5, 3, 1, 1), True), ((1024, 64, 32, 32, 5, 2, 0, 1), True),
    ((256, 64, 64, 64, 3, 1, 0, 1), True), ((32, 192, 28, 28, 5, 2, 0, 1), False),
])
def test_backward_path_choice(checker, case, one_pass):
    out = subprocess.run([checker, *map(str, case)], capture_output=True, text=True).stdout
    line = next(l for l in out.splitlines() if l.startswith("bwd:"))
    assert ("library picks one pass" in line) == one_pass, line
