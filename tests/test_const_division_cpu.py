"""The row scale fl(a/127) by division by a constant (CPU check of the rule).

The d = 128 decode kernel forms the INT8 row scale without a second IEEE
division: with y = RN(1/127), q0 = RN(a*y), r = a - q0*127 (exact, one fused
multiply-add) and q1 = RN(q0 + r*y) (one fused multiply-add), q1 is the
correctly rounded a/127 (Markstein's division by a constant).  Here the same
three operations run in C with fmaf() and are compared with IEEE division on
every subnormal, every float in [1, 2) and a strided sweep of all positive
finite floats.  (Run over all 2^31 positive floats the rule has no mismatch
for 127; for 448 it fails on subnormals, so FP8 rows keep IEEE division.)
"""
import ctypes
import os
import subprocess
import tempfile

SRC = r"""
#include <math.h>
#include <stdint.h>
#include <string.h>
static float f(uint32_t u) { float x; memcpy(&x, &u, 4); return x; }
static int one(float a, float b, float y) {
    const float q = a * y;
    const float q1 = fmaf(fmaf(-q, b, a), y, q);
    return q1 != a / b;
}
/* mismatches of the rule for b over u in [lo, hi) stepping by `step` */
long sweep(uint32_t lo, uint32_t hi, uint32_t step, float b) {
    const float y = 1.0f / b;
    long bad = 0;
    for (uint64_t u = lo; u < hi; u += step) bad += one(f((uint32_t)u), b, y);
    return bad;
}
"""


def _lib():
    d = tempfile.mkdtemp()
    src, so = os.path.join(d, "cdiv.c"), os.path.join(d, "cdiv.so")
    open(src, "w").write(SRC)
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
                    "-o", so, src, "-lm"], check=True)
    lib = ctypes.CDLL(so)
    lib.sweep.restype = ctypes.c_long
    lib.sweep.argtypes = [ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_float]
    return lib


def test_division_by_127_is_correctly_rounded():
    lib = _lib()
    assert lib.sweep(1, 0x00800000, 1, 127.0) == 0            # every subnormal
    assert lib.sweep(0x3F800000, 0x40000000, 1, 127.0) == 0   # every float in [1, 2)
    assert lib.sweep(1, 0x7F800000, 61, 127.0) == 0           # all binades, strided


def test_division_by_448_fails_on_subnormals():
    """Why FP8 rows keep IEEE division: the rule is not exact for 448."""
    lib = _lib()
    assert lib.sweep(1, 0x00800000, 1, 448.0) > 0
