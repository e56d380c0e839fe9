"""Real spherical harmonics (oracle; test infrastructure only).

Convention ("component" normalisation, the reading recorded in the design
notes): real basis, m = -l..l, z is the polar axis,
    sum_m Y_lm(n)^2 = 2l + 1,   Y_00 = 1,
    Y_l,m>0 ~ cos(m phi), Y_l,m<0 ~ sin(|m| phi), Condon-Shortley phase removed
by the real basis change in ``oracle.cg.real_basis``.

Construction: the complex solid harmonic r^l Y_l^m is the polynomial
    N_lm (-1)^m (x + i y)^m  sum_k a_k z^(l-m-2k) (x^2+y^2+z^2)^k,
where sum_k a_k t^(l-m-2k) is the m-th derivative of the Legendre polynomial
P_l(t) = 2^-l sum_k (-1)^k C(l,k) C(2l-2k, l) t^(l-2k). Real harmonics follow
from the real basis change; Y_lm(n) = P_lm(x,y,z) / r^l. Polynomial
coefficients are exact rationals times one square root per (l, m).
"""
from fractions import Fraction
from functools import lru_cache
from math import comb, factorial, sqrt

import numpy as np


def _padd(p, q, s=1):
    out = dict(p)
    for k, v in q.items():
        out[k] = out.get(k, 0) + s * v
    return {k: v for k, v in out.items() if v != 0}


def _pmul(p, q):
    out = {}
    for (a1, b1, c1), v1 in p.items():
        for (a2, b2, c2), v2 in q.items():
            k = (a1 + a2, b1 + b2, c1 + c2)
            out[k] = out.get(k, 0) + v1 * v2
    return {k: v for k, v in out.items() if v != 0}


def _ppow(p, n):
    out = {(0, 0, 0): Fraction(1)}
    for _ in range(n):
        out = _pmul(out, p)
    return out


def _legendre_deriv_coeffs(l, m):
    """Coefficients a_k of d^m/dt^m P_l(t) = sum_k a_k t^(l-m-2k)."""
    coeffs = {}
    for k in range(0, l // 2 + 1):
        c = Fraction((-1) ** k * comb(l, k) * comb(2 * l - 2 * k, l), 2 ** l)
        p = l - 2 * k
        if p < m:
            continue
        # d^m t^p = p!/(p-m)! t^(p-m)
        coeffs[k] = c * Fraction(factorial(p), factorial(p - m))
    return coeffs


@lru_cache(maxsize=None)
def _solid_complex_parts(l, m):
    """(Re, Im) rational polynomials of (x+iy)^m * sum_k a_k z^(l-m-2k) r^(2k), m >= 0."""
    re = {(0, 0, 0): Fraction(1)}
    im = {}
    # (x + i y)^m by repeated multiplication
    for _ in range(m):
        re, im = (_padd(_pmul(re, {(1, 0, 0): 1}), _pmul(im, {(0, 1, 0): 1}), -1),
                  _padd(_pmul(re, {(0, 1, 0): 1}), _pmul(im, {(1, 0, 0): 1})))
    r2 = {(2, 0, 0): 1, (0, 2, 0): 1, (0, 0, 2): 1}
    rad = {}
    for k, a in _legendre_deriv_coeffs(l, m).items():
        term = _pmul({(0, 0, l - m - 2 * k): a}, _ppow(r2, k))
        rad = _padd(rad, term)
    return _pmul(re, rad), _pmul(im, rad)


@lru_cache(maxsize=None)
def real_solid_polynomials(l):
    """List over m=-l..l of {(a,b,c): float} with Y_lm = P_lm(x,y,z) / r^l."""
    polys = []
    for m in range(-l, l + 1):
        am = abs(m)
        # component normalisation: sqrt(4 pi) * orthonormal N_lm
        n_lm = sqrt((2 * l + 1) * factorial(l - am) / factorial(l + am))
        re, im = _solid_complex_parts(l, am)
        if m == 0:
            p = {k: float(v) * n_lm for k, v in re.items()}
        elif m > 0:
            # sqrt(2) (-1)^m Re(Y^m); the (-1)^m of Y^m cancels
            p = {k: float(v) * n_lm * sqrt(2.0) for k, v in re.items()}
        else:
            p = {k: float(v) * n_lm * sqrt(2.0) for k, v in im.items()}
        polys.append(p)
    return polys


def _eval_poly(p, x, y, z):
    out = np.zeros(np.broadcast(x, y, z).shape, dtype=np.result_type(x, y, z, np.float64))
    for (a, b, c), v in p.items():
        out = out + v * x ** a * y ** b * z ** c
    return out


def _eval_poly_grad(p, x, y, z):
    gx = np.zeros(np.broadcast(x, y, z).shape, dtype=np.result_type(x, y, z, np.float64))
    gy = np.zeros_like(gx)
    gz = np.zeros_like(gx)
    for (a, b, c), v in p.items():
        if a:
            gx = gx + v * a * x ** (a - 1) * y ** b * z ** c
        if b:
            gy = gy + v * b * x ** a * y ** (b - 1) * z ** c
        if c:
            gz = gz + v * c * x ** a * y ** b * z ** (c - 1)
    return gx, gy, gz


def sh_real(l, vec):
    """Y_l(vec/|vec|) for vec [..., 3] (not necessarily unit). Returns [..., 2l+1].

    Works for complex input too (used by complex-step derivative checks):
    |vec| is sqrt(x^2+y^2+z^2) without conjugation, which is analytic.
    """
    vec = np.asarray(vec)
    x, y, z = vec[..., 0], vec[..., 1], vec[..., 2]
    r = np.sqrt(x * x + y * y + z * z)
    return np.stack([_eval_poly(p, x, y, z) / r ** l for p in real_solid_polynomials(l)], axis=-1)


def sh_real_grad(l, vec):
    """d Y_lm / d vec for vec [..., 3]. Returns [..., 2l+1, 3].

    Y = P / r^l  =>  dY/dv = grad P / r^l - l P v / r^(l+2).
    """
    vec = np.asarray(vec, dtype=np.float64)
    x, y, z = vec[..., 0], vec[..., 1], vec[..., 2]
    r2 = x * x + y * y + z * z
    r = np.sqrt(r2)
    outs = []
    for p in real_solid_polynomials(l):
        pv = _eval_poly(p, x, y, z)
        gx, gy, gz = _eval_poly_grad(p, x, y, z)
        rl = r ** l
        f = l * pv / (rl * r2)
        outs.append(np.stack([gx / rl - f * x, gy / rl - f * y, gz / rl - f * z], axis=-1))
    return np.stack(outs, axis=-2)
