"""The step kernel divides a group maximum by Qmax without a division
instruction: q0 = m * RN(1/Qmax), r = fma(-q0, Qmax, m), q = fma(r, RN(1/Qmax), q0)
(Markstein's correction for division by a constant; +inf keeps q0).  The
scale definition needs the correctly rounded binary32 quotient m / Qmax, so
the scheme must equal IEEE division for every non-negative m.

This checks the same operation sequence in C (gcc, no contraction, libm fmaf)
against the IEEE quotient: every subnormal and every pattern of the lowest
and highest binades, and a prime stride through the rest.  The full sweep of
all 2^31 + 1 patterns (about a minute on 8 cores) runs with QSTATE_DIV_FULL=1.
"""
from __future__ import annotations

import os
import subprocess
import tempfile

import numpy as np
import pytest

C_SRC = r"""
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
static float u2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static long long check(float d, float y, long long lo, long long hi, long long step) {
    long long bad = 0;
    #pragma omp parallel for reduction(+:bad) schedule(static)
    for (long long u = lo; u <= hi; u += step) {
        const float m = u2f((uint32_t)u);
        const float ref = m / d;
        const float q0 = m * y;
        const float r = fmaf(-q0, d, m);
        float q = fmaf(r, y, q0);
        if (r != r) q = q0;
        bad += f2u(q) != f2u(ref);
    }
    return bad;
}
int main(int argc, char** argv) {
    const float d = (float)atof(argv[1]);
    const float y = strtof(argv[2], NULL);
    const long long step = atoll(argv[3]);
    long long bad = 0;
    bad += check(d, y, 0, 0x01000000LL, 1);                     /* subnormals, lowest binade */
    bad += check(d, y, 0x7F000000LL, 0x7F800000LL, 1);          /* highest binade and +inf */
    bad += check(d, y, 0x01000001LL, 0x7EFFFFFFLL, step);
    printf("%lld\n", bad);
    return 0;
}
"""

# RN(1/Qmax) as written in the kernel
KERNEL_RECIPROCALS = {1: "0x1p+0", 7: "0x1.24924ap-3", 31: "0x1.08421p-5", 127: "0x1.020408p-7"}


@pytest.fixture(scope="module")
def checker():
    d = tempfile.mkdtemp(prefix="qdiv_")
    src, exe = os.path.join(d, "div.c"), os.path.join(d, "div")
    with open(src, "w") as f:
        f.write(C_SRC)
    subprocess.run(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-o", exe, src,
                    "-lm"], check=True)
    return exe


@pytest.mark.parametrize("qmax", [1, 7, 31, 127])
def test_kernel_reciprocal_constants(qmax):
    want = np.float32(1.0) / np.float32(qmax)
    assert np.float32(float.fromhex(KERNEL_RECIPROCALS[qmax])) == want


@pytest.mark.parametrize("qmax", [1, 7, 31, 127])
def test_division_by_qmax_is_correctly_rounded(checker, qmax):
    step = 1 if os.environ.get("QSTATE_DIV_FULL") == "1" else 127
    out = subprocess.run([checker, str(qmax), KERNEL_RECIPROCALS[qmax], str(step)],
                         capture_output=True, text=True, check=True).stdout
    assert int(out) == 0


def test_kernel_source_uses_these_constants():
    src = open(os.path.join(os.path.dirname(__file__), "..", "bit_recurrent_state_decode_b200",
                            "csrc", "qstate_kernel.cuh")).read()
    for q in (7, 31, 127):
        assert KERNEL_RECIPROCALS[q] + "f" in src
