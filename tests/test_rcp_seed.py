"""Host check of the kernels' reciprocal routine (csrc/rcp_seed.h): the same C
source the device code includes, compiled with gcc, against 1/a in double."""
import math
import os
import subprocess
import tempfile

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "gated_delta_rule_147_b200", "csrc")

PROG = r"""
#include <stdio.h>
#include "rcp_seed.h"
int main(void) {
    /* every mantissa of one binade, then a log-uniform sweep over the range the
       kernels use (reciprocals of decay factors 2^(+-115)) */
    double seed_max = 0, err_max = 0;
    for (unsigned m = 0; m < (1u << 23); ++m) {
        unsigned u = (127u << 23) | m; float a; memcpy(&a, &u, 4);
        double s = (double)gdr_rcp_seed(a) * a - 1.0, r = (double)gdr_rcp_newton3(a) * a - 1.0;
        if (fabs(s) > seed_max) seed_max = fabs(s);
        if (fabs(r) > err_max) err_max = fabs(r);
    }
    for (int i = 0; i < 4000000; ++i) {
        float a = (float)exp2(-115.0 + 230.0 * i / 4000000.0);
        double r = (double)gdr_rcp_newton3(a) * a - 1.0;
        if (fabs(r) > err_max) err_max = fabs(r);
    }
    printf("%.9e %.9e\n", seed_max, err_max);
    return 0;
}
"""


def test_seed_constant_is_the_derived_value():
    d = 5 - 2 * math.sqrt(6)
    src = open(os.path.join(HDR, "rcp_seed.h")).read()
    assert "0x7EF311C3u" in src
    assert round(2 ** 23 * (254 - d)) == 0x7EF311C3


def test_rcp_newton_error_bounds():
    with tempfile.TemporaryDirectory() as tmp:
        c = os.path.join(tmp, "rcp.c")
        exe = os.path.join(tmp, "rcp")
        open(c, "w").write(PROG)
        subprocess.run(["gcc", "-O2", "-I", HDR, "-o", exe, c, "-lm"], check=True)
        seed_max, err_max = map(float, subprocess.run([exe], check=True, capture_output=True,
                                                      text=True).stdout.split())
    d = 5 - 2 * math.sqrt(6)
    # the seed meets the derived bound d / 2 (and comes close to it)
    assert 0.9 * d / 2 < seed_max <= d / 2 + 1e-6
    # three Newton steps: within a few fp32 ulps of 1/a
    assert err_max < 4 * np.finfo(np.float32).eps
