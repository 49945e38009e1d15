"""Generate exp2_poly.cuh: 2^x on the FMA pipe for x <= 0, an alternative to
the MUFU ex2 instruction for a share of the exponentials of an exp-bound
epilogue.

Method (textbook, no vendor code):
  * range reduction in the manner of Cody and Waite: n = rint(x) by adding
    1.5 * 2^23 (the sum's low mantissa bits hold the rounded integer), then
    f = x - n, exact, in [-1/2, 1/2];
  * 2^f by a polynomial whose coefficients minimise the maximum RELATIVE
    error on [-1/2, 1/2] (Remez exchange, run here in float64), rounded to
    float32;
  * 2^n applied by adding n to the exponent field.
x is clamped to [-125, 0] first, so the result is always a normal float; for
x < -125 the result is about 2^-125 instead of a smaller value, an absolute
error below 3e-38.

Run from the repository root:  python -m sparse_attention_long_anchor_b200.csrc.gen_exp2_poly
(or directly as a script); it rewrites exp2_poly.cuh next to this file.
"""
import os

import numpy as np

DEGREES = (4, 5)
LO, HI = -0.5, 0.5


def _cheb_nodes(m):
    k = np.arange(m)
    return 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (2 * k + 1) / (2 * m))[::-1]


def remez_relative(deg, iters=60):
    """Coefficients c[0..deg] (ascending) of the polynomial p minimising
    max |p(f) / 2^f - 1| on [LO, HI], and that maximum."""
    ref = np.sort(_cheb_nodes(deg + 2))
    grid = np.linspace(LO, HI, 200001)
    c = None
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i  ->  linear in (c, E)
        A = np.zeros((deg + 2, deg + 2))
        for i, x in enumerate(ref):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** ref)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: the extremum of each sign-alternating run of err
        sign = np.sign(err)
        sign[sign == 0] = 1
        cuts = np.flatnonzero(np.diff(sign)) + 1
        runs = np.split(np.arange(grid.size), cuts)
        ext = np.array([r[np.argmax(np.abs(err[r]))] for r in runs])
        if ext.size < deg + 2:
            break
        if ext.size > deg + 2:   # keep the deg + 2 largest, in order, preserving alternation
            keep = np.sort(np.argsort(-np.abs(err[ext]))[:deg + 2])
            ext = ext[keep]
        new_ref = grid[ext]
        if np.allclose(new_ref, ref, atol=1e-12):
            break
        ref = new_ref
    err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
    return c, float(np.max(np.abs(err)))


def f32(x):
    return np.float32(x)


def emulate(x, coeffs32):
    """The header's evaluation, step by step, in float32 arithmetic (each
    fused multiply-add rounded once: the float64 product of two float32 values
    is exact)."""
    x = np.minimum(np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125.0)), np.float32(0.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n_f = (t - magic).astype(np.float32)
    f = (x - n_f).astype(np.float32)
    p = np.full_like(f, coeffs32[-1])
    for ck in coeffs32[-2::-1]:
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(ck)).astype(np.float32)
    bits = p.view(np.int32) + (n_f.astype(np.int32) << 23)
    return bits.view(np.float32)


def fitted():
    """{degree: (float32 coefficients ascending, float64 fit error)}"""
    out = {}
    for deg in DEGREES:
        c, e = remez_relative(deg)
        out[deg] = ([f32(v) for v in c], e)
    return out


def measured_bound(coeffs32, samples=1 << 21, seed=0):
    """Max relative error of the float32 evaluation over a dense sample of
    [-125, 0] plus the half-integer and integer points."""
    rng = np.random.default_rng(seed)
    xs = np.concatenate([rng.uniform(-125.0, 0.0, samples),
                         np.arange(-125.0, 0.5, 0.5), np.linspace(-1.0, 0.0, 4097)]).astype(np.float32)
    got = emulate(xs, coeffs32).astype(np.float64)
    ref = np.exp2(np.maximum(xs.astype(np.float64), -125.0))
    return float(np.max(np.abs(got / ref - 1.0)))


def header_text(fit):
    lines = [
        "// 2^x on the FMA pipe for x <= 0 (written by gen_exp2_poly.py; do not edit).",
        "// Cody-Waite style reduction n = rint(x), f = x - n in [-1/2, 1/2]; 2^f by a",
        "// polynomial minimising the maximum relative error (Remez exchange),",
        "// coefficients rounded to float32; 2^n added to the exponent field.  x is",
        "// clamped to [-125, 0], so the result is a normal float.",
        "#pragma once",
        "",
        "namespace kascade {",
        "",
    ]
    for deg, (c32, fit_err) in fit.items():
        bound = measured_bound(c32)
        lines.append(f"// degree {deg}: fit error {fit_err:.3e}, float32 evaluation error <= {bound:.3e} (sampled)")
        lines.append(f"__device__ __forceinline__ float exp2_poly{deg}(float x) {{")
        lines.append("  x = fminf(fmaxf(x, -125.0f), 0.0f);")
        lines.append("  const float t = x + 12582912.0f;   // 1.5 * 2^23: low mantissa bits = rint(x)")
        lines.append("  const float n = t - 12582912.0f;")
        lines.append("  const float f = x - n;")
        lines.append(f"  float p = {float(c32[-1])!r}f;")
        for ck in c32[-2::-1]:
            lines.append(f"  p = fmaf(p, f, {float(ck)!r}f);")
        lines.append("  return __int_as_float(__float_as_int(p) + (__float_as_int(t) - 0x4B400000) * (1 << 23));")
        lines.append("}")
        lines.append("")
    lines.append("}  // namespace kascade")
    return "\n".join(lines) + "\n"


def main():
    fit = fitted()
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "exp2_poly.cuh")
    with open(path, "w") as fh:
        fh.write(header_text(fit))
    for deg, (c32, e) in fit.items():
        print(f"degree {deg}: fit {e:.3e}, float32 evaluation {measured_bound(c32):.3e}")
    print("wrote", path)


if __name__ == "__main__":
    main()
