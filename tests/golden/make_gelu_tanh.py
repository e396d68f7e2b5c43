"""Write gelu_tanh.json: the tanh form of GELU worked from its definition in
exact decimal arithmetic (40 significant digits), step by step.

The tanh form is  GELU_tanh(z) = z/2 * (1 + tanh(sqrt(2/pi) * (z + 0.044715 z^3)))
(Hendrycks and Gimpel, "Gaussian Error Linear Units", 2016, section 2).  The
codec offers it as the alternative to exact GELU z * Phi(z).

This script does not use the oracle or the CUDA library, nor any floating-point
library routine: pi comes from Machin's formula, tanh from the decimal
exponential, and every intermediate value is written out so that a reader can
redo each step by hand.  Run it from any directory:
    python tests/golden/make_gelu_tanh.py
"""
import decimal
import json
import os
from decimal import Decimal as Dec

decimal.getcontext().prec = 60
A = Dec("0.044715")
ZS = ["-3", "-1", "-0.5", "0.5", "1", "2", "3"]


def atan_inv(x: int) -> Dec:
    """atan(1/x) by its alternating power series."""
    x2 = Dec(x) * Dec(x)
    term = Dec(1) / Dec(x)
    total, n = Dec(0), 0
    while True:
        t = term / (2 * n + 1)
        if abs(t) < Dec(10) ** -58:
            break
        total += t if n % 2 == 0 else -t
        term /= x2
        n += 1
    return total


def main():
    pi = 16 * atan_inv(5) - 4 * atan_inv(239)          # Machin (1706)
    c = (Dec(2) / pi).sqrt()
    rows = []
    for zs in ZS:
        z = Dec(zs)
        poly = z + A * z * z * z                          # exact in decimal
        y = c * poly
        e2y = (2 * y).exp()
        th = (e2y - 1) / (e2y + 1)
        val = z / 2 * (1 + th)
        rows.append({"z": float(z), "z_plus_a_z3": str(poly), "y": f"{y:.40g}", "tanh_y": f"{th:.40g}",
                     "gelu_tanh": f"{val:.40g}"})
    doc = {
        "about": "GELU in its tanh form, z/2 (1 + tanh(sqrt(2/pi) (z + 0.044715 z^3))) (Hendrycks and Gimpel "
                 "2016, section 2), worked from the definition in 60-digit decimal arithmetic by "
                 "tests/golden/make_gelu_tanh.py: pi by Machin's formula, sqrt(2/pi), the cubic "
                 "(exact in decimal), y = sqrt(2/pi) times the cubic, tanh y = (e^2y - 1)/(e^2y + 1), then "
                 "z/2 (1 + tanh y).  Values printed to 40 significant digits.",
        "pi": f"{pi:.40g}",
        "sqrt_2_over_pi": f"{c:.40g}",
        "a": str(A),
        "rows": rows,
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "gelu_tanh.json")
    with open(path, "w") as f:
        json.dump(doc, f, indent=1)
        f.write("\n")
    print(path)


if __name__ == "__main__":
    main()
