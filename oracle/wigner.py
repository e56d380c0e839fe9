"""Wigner D matrices (oracle; test infrastructure only).

Used only by the equivariance pins: a second, independent route to how real
spherical harmonics and real-basis CG tensors transform under rotations.

Complex D from Wigner's small-d formula,
    D^l_{m'm}(a, b, g) = exp(-i m' a) d^l_{m'm}(b) exp(-i m g),
for R = Rz(a) Ry(b) Rz(g). Complex harmonics then satisfy
    Y^m(R n) = sum_m' conj(D^l_{m m'}(R)) Y^m'(n),
so in the real basis D_real(R) = Q_l conj(D^l(R)) Q_l^dagger.
"""
from math import factorial, sqrt

import numpy as np

from .cg import real_basis


def small_d(l, beta):
    d = np.zeros((2 * l + 1, 2 * l + 1))
    cb, sb = np.cos(beta / 2.0), np.sin(beta / 2.0)
    for mp in range(-l, l + 1):
        for m in range(-l, l + 1):
            pref = sqrt(factorial(l + mp) * factorial(l - mp) * factorial(l + m) * factorial(l - m))
            acc = 0.0
            for s in range(0, 2 * l + 1):
                a, b, c, e = l + m - s, s, mp - m + s, l - mp - s
                if min(a, b, c, e) < 0:
                    continue
                acc += ((-1) ** (mp - m + s) / (factorial(a) * factorial(b) * factorial(c) * factorial(e))
                        * cb ** (2 * l + m - mp - 2 * s) * sb ** (mp - m + 2 * s))
            d[mp + l, m + l] = pref * acc
    return d


def wigner_D_complex(l, alpha, beta, gamma):
    ms = np.arange(-l, l + 1)
    return (np.exp(-1j * ms * alpha)[:, None] * small_d(l, beta) * np.exp(-1j * ms * gamma)[None, :])


def wigner_D_real(l, alpha, beta, gamma):
    q = real_basis(l)
    d = q @ wigner_D_complex(l, alpha, beta, gamma).conj() @ q.conj().T
    assert np.abs(d.imag).max() < 1e-12
    return d.real


def rotation_matrix(alpha, beta, gamma):
    """R = Rz(alpha) Ry(beta) Rz(gamma) acting on column vectors."""
    def rz(t):
        c, s = np.cos(t), np.sin(t)
        return np.array([[c, -s, 0.0], [s, c, 0.0], [0.0, 0.0, 1.0]])

    def ry(t):
        c, s = np.cos(t), np.sin(t)
        return np.array([[c, 0.0, s], [0.0, 1.0, 0.0], [-s, 0.0, c]])

    return rz(alpha) @ ry(beta) @ rz(gamma)


def euler_angles(rot):
    """Inverse of ``rotation_matrix`` (ZYZ), for a proper rotation matrix."""
    beta = np.arccos(np.clip(rot[2, 2], -1.0, 1.0))
    if abs(np.sin(beta)) > 1e-12:
        alpha = np.arctan2(rot[1, 2], rot[0, 2])
        gamma = np.arctan2(rot[2, 1], -rot[2, 0])
    else:  # gimbal lock: only alpha + gamma is defined
        alpha = np.arctan2(rot[1, 0], rot[0, 0]) if rot[2, 2] > 0 else np.arctan2(-rot[1, 0], -rot[0, 0])
        gamma = 0.0
    return alpha, beta, gamma


def random_rotation(rng):
    """Haar-random proper rotation (QR of a Gaussian matrix, det fixed to +1)."""
    q, r = np.linalg.qr(rng.standard_normal((3, 3)))
    q = q * np.sign(np.diag(r))[None, :]
    if np.linalg.det(q) < 0:
        q[:, 0] = -q[:, 0]
    return q
