"""Fits the polynomial of the kernel's software exp2 (run once; prints the coefficients).

Software exp2 on the FMA pipes takes the load off the MUFU unit (page "FlashAttention 4:
Γρηγορότερη και Αποδοτική σε Μνήμη Προσοχή για LLMs", section "Αποκορύφωση Λογισμικού
μέσω Πυρήνων CUDA": a cubic polynomial evaluated on the CUDA cores instead of the SFUs).
The method here is the textbook one, fitted from scratch:

  2^x = 2^j * 2^f,  j = round(x),  f = x - j in [-1/2, 1/2]   (Cody-Waite range reduction)
  2^f ~ c0 + c1 f + c2 f^2 + c3 f^3                            (near-minimax in relative error)

The fit is a Lawson-weighted least-squares iteration on a dense grid (it converges to the
equioscillating minimax polynomial), done in float64 and then rounded to float32.

    python -m tiled_attention_14_b200.fit_exp2_poly
"""
from __future__ import annotations

import numpy as np

DEGREE = 3


def fit(degree: int = DEGREE, iters: int = 200) -> np.ndarray:
    f = np.cos(np.linspace(0.0, np.pi, 4001)) * 0.5          # Chebyshev-spaced points on [-1/2, 1/2]
    target = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / target[:, None]   # relative error rows
    b = np.ones_like(f)
    w = np.ones_like(f)
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        err = np.abs(A @ c - b)
        w = w * err
        w /= w.sum()
    return c


def max_rel_error_f32(c32: np.ndarray) -> float:
    """Max relative error of the float32 Horner evaluation over [-1/2, 1/2]."""
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = np.full_like(f, c32[-1])
    for k in range(len(c32) - 2, -1, -1):
        p = (p * f + c32[k]).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    c = fit()
    c32 = c.astype(np.float32)
    print("coefficients (float32):", [float(x) for x in c32])
    print("hex:", [hex(np.float32(x).view(np.uint32)) for x in c32])
    print("max relative error (float32 Horner):", max_rel_error_f32(c32))
