"""bench.py's metric arithmetic (CPU): the modeled bytes behind the GB/s
figures and the multiply-add count behind the ALU roofline, each checked
against an independent count.

- Bytes: every call reads its activation input(s) and writes its output once
  (forward: x -> y; input gradient: dy -> dx; weight gradient: x and dy in),
  plus the parameters (read by every call, and the gradients written by the
  weight gradient); the parameter sizes are taken from the tensors the input
  recipe builds, not from a formula.
- Multiply-adds: one k x k tap per output of the base conv and of every
  subband conv, counted level by level from the subband sizes.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from wtconv_inputs import NAMED, make_inputs, sweep_cases  # noqa: E402

PARAMS = ("base_w", "base_b", "base_scale", "wt_w", "wt_scale")


def param_bytes_from_tensors(case):
    inp = make_inputs(case.with_(B=1, C=case.C))  # parameter shapes do not depend on B
    return sum(inp[k].numel() * 4 for k in PARAMS)


def fmas_by_levels(case):
    per_plane = case.H * case.W * case.k * case.k
    for l in range(case.L):
        per_plane += 4 * (case.H >> (l + 1)) * (case.W >> (l + 1)) * case.k * case.k
    return case.B * case.C * per_plane


@pytest.mark.parametrize("name", ["stage1", "stage2", "train_bf16"])
def test_modeled_bytes_per_call(name):
    case = NAMED[name]
    act = case.B * case.C * case.H * case.W * case.esize
    P = param_bytes_from_tensors(case)
    mb = bench.modeled_bytes(case)
    assert mb == {"fwd": 2 * act + P, "bwd_in": 2 * act + P, "bwd_w": 2 * act + 2 * P}


def test_stage1_step_bytes_value():
    # 32 x 96 x 56 x 56 fp32 activations, k = 5, L = 3: 231,731,712 bytes per step.
    assert sum(bench.modeled_bytes(NAMED["stage1"]).values()) == 231_731_712


@pytest.mark.parametrize("case", [NAMED["stage1"], NAMED["stage2"], NAMED["train_bf16"]]
                         + [c for c in sweep_cases() if c.name.startswith(("sweep007", "sweep063", "sweep127"))],
                         ids=lambda c: c.name)
def test_conv_fmas_match_level_count(case):
    assert bench.conv_fmas(case) == pytest.approx(fmas_by_levels(case), rel=0, abs=0.5)


def test_stage1_flops_per_launch():
    # 181,300 multiply-adds per 56 x 56 plane (78,400 base + 78,400 + 19,600 + 4,900 subband), 3,072 planes.
    assert fmas_by_levels(NAMED["stage1"]) == 181_300 * 3072
    assert 2 * bench.conv_fmas(NAMED["stage1"]) == 1_113_907_200
