"""Radial basis and cutoff envelope (oracle; test infrastructure only).

Reading of the workload description (Bessel radial basis with a p = 6
polynomial cutoff, projected through a small weight matrix): the NequIP-style
basis with fixed frequencies,
    B_n(d) = (2 / r_c) sin(n pi d / r_c) / d,          n = 1..n_basis,
times the polynomial envelope, t = d / r_c,
    u(t) = 1 - (p+1)(p+2)/2 t^p + p(p+2) t^(p+1) - p(p+1)/2 t^(p+2)   (t < 1),
    u(t) = 0                                                          (t >= 1).
"""
import numpy as np

P_ENVELOPE = 6


def envelope(t, p=P_ENVELOPE):
    t = np.asarray(t)
    val = (1.0 - (p + 1) * (p + 2) / 2.0 * t ** p + p * (p + 2) * t ** (p + 1)
           - p * (p + 1) / 2.0 * t ** (p + 2))
    return np.where(np.real(t) < 1.0, val, 0.0 * val)


def envelope_deriv(t, p=P_ENVELOPE):
    """du/dt = -p(p+1)(p+2)/2 t^(p-1) (1 - t)^2 for t < 1, else 0."""
    t = np.asarray(t)
    val = -p * (p + 1) * (p + 2) / 2.0 * t ** (p - 1) * (1.0 - t) ** 2
    return np.where(np.real(t) < 1.0, val, 0.0 * val)


def bessel(d, n_basis, r_cut):
    """B_n(d) for d [...] -> [..., n_basis]."""
    d = np.asarray(d)[..., None]
    n = np.arange(1, n_basis + 1)
    return (2.0 / r_cut) * np.sin(n * np.pi * d / r_cut) / d


def bessel_deriv(d, n_basis, r_cut):
    d = np.asarray(d)[..., None]
    k = np.arange(1, n_basis + 1) * np.pi / r_cut
    return (2.0 / r_cut) * (k * np.cos(k * d) / d - np.sin(k * d) / (d * d))


def radial(d, n_basis, r_cut, p=P_ENVELOPE):
    """R_n(d) = B_n(d) u(d / r_c)  ->  [..., n_basis]."""
    return bessel(d, n_basis, r_cut) * envelope(np.asarray(d) / r_cut, p)[..., None]


def radial_deriv(d, n_basis, r_cut, p=P_ENVELOPE):
    d = np.asarray(d)
    u = envelope(d / r_cut, p)[..., None]
    du = envelope_deriv(d / r_cut, p)[..., None] / r_cut
    return bessel_deriv(d, n_basis, r_cut) * u + bessel(d, n_basis, r_cut) * du
