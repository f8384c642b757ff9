"""Writes gelu_tanh.txt: the tanh form of GELU at a few points, in 40-digit
decimal arithmetic, straight from the published formula

    gelu_tanh(y) = 0.5 y (1 + tanh(sqrt(2 / pi) (y + 0.044715 y^3)))

(Hendrycks & Gimpel, "Gaussian Error Linear Units", the tanh approximation;
the tiny TP MLP workload applies this form between c_fc and c_proj).  Only the
standard library's decimal module is used, not numpy or the oracle, so the
values pin the oracle's float64 implementation from outside it.

    python tests/golden/make_gelu_tanh.py > tests/golden/gelu_tanh.txt
"""
from decimal import Decimal, getcontext

getcontext().prec = 40


def arctan_inv(n: int) -> Decimal:
    """arctan(1/n) by its Taylor series."""
    x = Decimal(1) / n
    x2 = x * x
    term, total, k = x, x, 1
    eps = Decimal(10) ** (-(getcontext().prec + 2))
    while abs(term) > eps:
        term *= -x2
        k += 2
        total += term / k
    return total


def pi() -> Decimal:
    """Machin's formula: pi = 16 arctan(1/5) - 4 arctan(1/239)."""
    return 16 * arctan_inv(5) - 4 * arctan_inv(239)


def tanh(z: Decimal) -> Decimal:
    e = (2 * z).exp()
    return (e - 1) / (e + 1)


def gelu_tanh(y: Decimal) -> Decimal:
    c = (Decimal(2) / pi()).sqrt()
    return Decimal("0.5") * y * (1 + tanh(c * (y + Decimal("0.044715") * y ** 3)))


POINTS = ["-3.0", "-1.5", "-0.5", "0.1", "0.7", "1.0", "2.0", "4.5"]

if __name__ == "__main__":
    print("# GELU, tanh form, 0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3)))")
    print("# (Hendrycks & Gimpel, tanh approximation), 40-digit decimal arithmetic;")
    print("# written by tests/golden/make_gelu_tanh.py (standard library only).")
    print("# columns: y gelu_tanh(y)")
    for p in POINTS:
        print(p, format(gelu_tanh(Decimal(p)), ".25e"))
