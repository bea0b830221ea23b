"""The FMA-pipe 2^x of the kernels (exp2_poly2 in csrc/sm100_ptx.cuh): its
four coefficients, read from the header itself, are a minimax (Remez) fit of
2^f on [-1/2, 1/2] with p(0) = 1, checked in fp64 on the CPU:

* the relative error p(f) / 2^f - 1 stays below 3.6e-6;
* it equioscillates: five local extrema of alternating sign and (to 2%) equal
  magnitude, the characterisation of the best approximation with four free
  coefficients (Chebyshev's alternation theorem);
* every small change of one coefficient makes the maximum error larger.

The GPU self-test (tests/test_selftest_gpu.py) then checks the full
evaluation, reduction included, against exp2 on the device."""
import os
import re

import numpy as np

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "exact_io_aware_52_b200", "csrc",
                      "sm100_ptx.cuh")


def coefficients():
    """(c1, c2, c3, c4) of p(f) = 1 + c1 f + c2 f^2 + c3 f^3 + c4 f^4 as written in
    the Horner steps of exp2_poly2 (highest degree first)."""
    src = open(HEADER).read()
    body = src[src.index("float2 exp2_poly2("):]
    body = body[:body.index("\n}\n")]
    lits = re.findall(r"make_float2\(([0-9.eE+-]+)f, \1f\)", body)
    vals = [float(x) for x in lits]
    # the literals in order: clamp and magic constants, then c4, c3, c2, c1, 1
    horner = [v for v in vals if 0.0 < v < 1.0]
    assert len(horner) == 4, vals
    c4, c3, c2, c1 = horner
    return c1, c2, c3, c4


def rel_error(c, f):
    c1, c2, c3, c4 = c
    p = 1.0 + f * (c1 + f * (c2 + f * (c3 + f * c4)))
    return p / np.exp2(f) - 1.0


F = np.linspace(-0.5, 0.5, 400001)


def test_error_bound():
    assert np.abs(rel_error(coefficients(), F)).max() <= 3.6e-6


def extrema(e):
    """The signed extreme values of e between its sign changes (the error's
    alternation points), endpoints included."""
    out = []
    start = 0
    s = np.sign(e)
    for i in range(1, len(e) + 1):
        if i == len(e) or (s[i] != s[start] and s[i] != 0):
            seg = e[start:i]
            out.append(seg[np.argmax(np.abs(seg))])
            start = i
    return np.array(out)


def test_equioscillation():
    e = rel_error(coefficients(), F)
    emax = np.abs(e).max()
    ext = extrema(e)
    big = ext[np.abs(ext) >= 0.98 * emax]
    assert len(big) >= 5, ext
    assert np.all(np.sign(big[1:]) != np.sign(big[:-1])), ext


def test_no_nearby_coefficients_do_better():
    """A change of 1e-4 (relative) in any coefficient makes the maximum error
    larger; a change of 1e-5 cannot make it smaller by more than 0.5% (the
    coefficients are the fit rounded to float32)."""
    c = np.array(coefficients())
    base = np.abs(rel_error(c, F)).max()
    for i in range(4):
        for rel in (1e-4, -1e-4):
            cc = c.copy()
            cc[i] *= 1.0 + rel
            assert np.abs(rel_error(cc, F)).max() > base, (i, rel)
        for rel in (1e-5, -1e-5):
            cc = c.copy()
            cc[i] *= 1.0 + rel
            assert np.abs(rel_error(cc, F)).max() > 0.995 * base, (i, rel)
