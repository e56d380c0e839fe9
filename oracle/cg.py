"""Clebsch-Gordan coefficients (oracle; test infrastructure only).

Complex CG from Racah's closed form in exact rational arithmetic, then the
change to the real spherical-harmonic basis. The pages cite the coupling only
by name ("Fast and Accurate Foundation Models for Equivariant MLIPs", section
VII: tensor products with irreps parity restricted to that of the spherical
harmonics; "FlashCart", Table C1: sparse Clebsch-Gordan coupling); the closed
form and the real basis are the textbook ones (Condon-Shortley phase).
"""
from fractions import Fraction
from functools import lru_cache
from math import factorial, sqrt

import numpy as np


def _f(n):
    return factorial(n)


@lru_cache(maxsize=None)
def cg_complex(l1, m1, l2, m2, l3, m3):
    """<l1 m1 l2 m2 | l3 m3> for the complex (Condon-Shortley) basis.

    Racah's formula: a square-root prefactor times a finite alternating sum.
    The squared prefactor and the sum are exact Fractions; one float sqrt at
    the end.
    """
    if m1 + m2 != m3:
        return 0.0
    if not (abs(l1 - l2) <= l3 <= l1 + l2):
        return 0.0
    if abs(m1) > l1 or abs(m2) > l2 or abs(m3) > l3:
        return 0.0
    pref2 = Fraction((2 * l3 + 1) * _f(l3 + l1 - l2) * _f(l3 - l1 + l2) * _f(l1 + l2 - l3),
                     _f(l1 + l2 + l3 + 1))
    pref2 *= (_f(l3 + m3) * _f(l3 - m3) * _f(l1 - m1) * _f(l1 + m1) * _f(l2 - m2) * _f(l2 + m2))
    total = Fraction(0)
    for k in range(0, l1 + l2 + l3 + 1):
        d = [k, l1 + l2 - l3 - k, l1 - m1 - k, l2 + m2 - k, l3 - l2 + m1 + k, l3 - l1 - m2 + k]
        if min(d) < 0:
            continue
        den = 1
        for v in d:
            den *= _f(v)
        total += Fraction((-1) ** k, den)
    if total == 0:
        return 0.0
    sign = 1.0 if total > 0 else -1.0
    # value = sqrt(pref2) * total = sign * sqrt(pref2 * total^2)
    return sign * sqrt(float(pref2 * total * total))


def real_basis(l):
    """Unitary Q_l with real SH = Q_l @ complex SH (rows and columns m=-l..l).

    m > 0 : Y_real =  ((-1)^m Y^m + Y^-m) / sqrt(2)   (proportional to cos(m phi))
    m < 0 : Y_real = i (Y^-|m| - (-1)^|m| Y^|m|) / sqrt(2)  (proportional to sin(|m| phi))
    m = 0 : Y_real = Y^0
    """
    q = np.zeros((2 * l + 1, 2 * l + 1), dtype=np.complex128)
    s = 1.0 / sqrt(2.0)
    q[l, l] = 1.0
    for m in range(1, l + 1):
        q[l + m, l + m] = (-1) ** m * s
        q[l + m, l - m] = s
        q[l - m, l - m] = 1j * s
        q[l - m, l + m] = -1j * (-1) ** m * s
    return q


@lru_cache(maxsize=None)
def _cg_complex_tensor(l1, l2, l3):
    c = np.zeros((2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1))
    for m1 in range(-l1, l1 + 1):
        for m2 in range(-l2, l2 + 1):
            m3 = m1 + m2
            if abs(m3) <= l3:
                c[m1 + l1, m2 + l2, m3 + l3] = cg_complex(l1, m1, l2, m2, l3, m3)
    return c


@lru_cache(maxsize=None)
def cg_real(l1, l2, l3):
    """Real-basis CG tensor C[m1, m2, m3] (indices offset by l), float64.

    With T[a,b,c] = sum conj(Q1[a,m1]) conj(Q2[b,m2]) Q3[c,m3] C_complex[m1,m2,m3], the vector
    z_c = sum_ab T[a,b,c] x_a y_b couples real-basis vectors the way the complex CG couples
    complex ones. For l1+l2+l3 even T is real and is returned as it is (the only case that
    irreps with the harmonics' parity use). For l1+l2+l3 odd T is purely imaginary, T = i T',
    and the coupling of real vectors is the real tensor T' (the imaginary part), an
    antisymmetric coupling such as the cross product for 1 x 1 -> 1; its overall sign is a
    convention that a path weight absorbs.
    """
    if not (abs(l1 - l2) <= l3 <= l1 + l2):
        raise ValueError("triangle rule violated")
    cc = _cg_complex_tensor(l1, l2, l3)
    q1, q2, q3 = real_basis(l1), real_basis(l2), real_basis(l3)
    r = np.einsum("ai,bj,ck,ijk->abc", q1.conj(), q2.conj(), q3, cc)
    if (l1 + l2 + l3) % 2 == 0:
        assert np.abs(r.imag).max() < 1e-13, (l1, l2, l3)
        out = r.real.copy()
    else:
        assert np.abs(r.real).max() < 1e-13, (l1, l2, l3)
        out = r.imag.copy()
    out[np.abs(out) < 1e-14] = 0.0
    out.setflags(write=False)
    return out
