"""Every plausible mistake planted in the oracle is caught by a pin.

Each mutant is a textual edit of a copy of oracle/wtconv_oracle.c (a wrong
sign, a transposed kernel, a misplaced bias or scale, a wrong recursion, a
missing adjoint rotation...), compiled on the CPU into a temporary library.
The test runs every pin of oracle_pins.py against it and requires at least
one to fail.  The committed oracle itself passes all pins (test_oracle.py).
"""
import os
import tempfile

import pytest

import oracle as orc_pkg
from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(orc_pkg.__file__), "wtconv_oracle.c")

MUTANTS = {
    # analysis computes LH with the column signs
    "dwt2_lh_sign": ("S[1 * m + o] = (a + b - c - d) / 2.0;", "S[1 * m + o] = (a - b + c - d) / 2.0;"),
    # synthesis swaps the roles of LH and HL in one output
    "iwt2_swap": ("X[(size_t)(2 * i) * nw + 2 * j + 1] = (ll + lh - hl - hh) / 2.0;",
                  "X[(size_t)(2 * i) * nw + 2 * j + 1] = (ll - lh + hl - hh) / 2.0;"),
    # orthonormal factor dropped in the analysis
    "dwt2_norm": ("S[0 * m + o] = (a + b + c + d) / 2.0;", "S[0 * m + o] = (a + b + c + d) / 4.0;"),
    # kernel transposed
    "dwconv_transposed": ("acc += w[u * k + v] * X[(size_t)r * nw + q];",
                          "acc += w[v * k + u] * X[(size_t)r * nw + q];"),
    # adjoint without the 180-degree rotation
    "adjoint_not_rotated": ("int r = i - u + p;", "int r = i + u - p;"),
    # bias added after the scale
    "bias_outside_scale": ("yp[i] = base_scale[c] * (yp[i] + base_b[c]);",
                           "yp[i] = base_scale[c] * yp[i] + base_b[c];"),
    # coarser reconstruction added into LH instead of LL (forward)
    "coarse_into_lh": ("for (size_t i = 0; i < m; ++i) S[i] += z[i]; /* coarser reconstruction into LL */",
                       "for (size_t i = 0; i < m; ++i) S[m + i] += z[i];"),
    # subband scale not applied in the forward
    "no_subband_scale": ("                for (size_t i = 0; i < m; ++i) dst[i] *= a;\n            }\n        }\n\n        /* synthesis",
                         "            }\n        }\n\n        /* synthesis"),
    # recursion on LH instead of the raw LL
    "recurse_on_lh": ("cur = S; /* S_{l,LL}: the raw approximation recurses */",
                      "cur = S + (size_t)(nh / 2) * (nw / 2);"),
    # backward: coarser gradient added into LH
    "bwd_coarse_into_lh": ("for (size_t i = 0; i < m; ++i) S[i] += g[i];", "for (size_t i = 0; i < m; ++i) S[m + i] += g[i];"),
    # backward input without the base scale
    "bwd_no_base_scale": ("for (size_t i = 0; i < plane; ++i) dxp[i] *= base_scale[c];", ""),
    # weight gradient without the subband scale factor
    "dwtw_no_scale": ("d_wt_w[pi * kk + t] = wt_scale[pi] * gw[((size_t)l * 4 + s) * kk + t];",
                      "d_wt_w[pi * kk + t] = gw[((size_t)l * 4 + s) * kk + t];"),
    # base-scale gradient without the bias term
    "dbs_no_bias": ("dbs += gp[i] * (conv[i] + base_b[c]);", "dbs += gp[i] * conv[i];"),
    # base-weight gradient correlates with the wrong shift direction
    "dbw_shift_sign": ("int r = h + u - p;", "int r = h - u + p;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    src = open(SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = src.replace(old, new, 1)
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "mutant.c")
        so = os.path.join(d, "libmutant.so")
        open(c, "w").write(mutated)
        orc_pkg.compile_oracle(c, so)
        orc = orc_pkg.Oracle(orc_pkg.load_library(so))
        failed = []
        for pin in ALL_PINS:
            try:
                pin(orc)
            except AssertionError:
                failed.append(pin.__name__)
        assert failed, f"mutant {name} passed every pin"
