"""Pins for the oracle's spherical harmonics, Wigner D and radial basis (CPU only)."""
import numpy as np
import pytest
import scipy.special as sps
from numpy.polynomial import legendre

from oracle.cg import real_basis
from oracle.radial import bessel, bessel_deriv, envelope, envelope_deriv, radial, radial_deriv
from oracle.sh import sh_real, sh_real_grad
from oracle.wigner import euler_angles, random_rotation, rotation_matrix, wigner_D_real


def _unit(rng, n):
    v = rng.standard_normal((n, 3))
    return v / np.linalg.norm(v, axis=1, keepdims=True)


@pytest.mark.parametrize("l", range(5))
def test_sh_matches_scipy_complex_harmonics(l):
    # scipy's sph_harm_y (orthonormal, Condon-Shortley) through the real basis, times sqrt(4 pi)
    rng = np.random.default_rng(l)
    v = rng.standard_normal((64, 3)) * rng.uniform(0.3, 4.0, size=(64, 1))
    n = v / np.linalg.norm(v, axis=1, keepdims=True)
    theta, phi = np.arccos(n[:, 2]), np.arctan2(n[:, 1], n[:, 0])
    yc = np.stack([sps.sph_harm_y(l, m, theta, phi) for m in range(-l, l + 1)], axis=-1)
    yr = (real_basis(l) @ yc.T).T * np.sqrt(4 * np.pi)
    assert np.abs(yr.imag).max() < 1e-13
    assert np.abs(yr.real - sh_real(l, v)).max() < 1e-13


@pytest.mark.parametrize("l", range(5))
def test_sh_addition_theorem_and_norm(l):
    rng = np.random.default_rng(10 + l)
    a, b = _unit(rng, 50), _unit(rng, 50)
    lhs = (sh_real(l, a) * sh_real(l, b)).sum(-1)
    pl = legendre.legval((a * b).sum(-1), [0] * l + [1])
    assert np.abs(lhs - (2 * l + 1) * pl).max() < 1e-12
    assert np.abs((sh_real(l, a) ** 2).sum(-1) - (2 * l + 1)).max() < 1e-12
    if l == 0:
        assert np.all(sh_real(0, a) == 1.0)


@pytest.mark.parametrize("l", range(4))
def test_sh_equivariance_and_parity(l):
    rng = np.random.default_rng(20 + l)
    v = rng.standard_normal((40, 3))
    for _ in range(3):
        rot = random_rotation(rng)
        a, b, g = euler_angles(rot)
        assert np.abs(rotation_matrix(a, b, g) - rot).max() < 1e-12
        d = wigner_D_real(l, a, b, g)
        assert np.abs(sh_real(l, v @ rot.T) - sh_real(l, v) @ d.T).max() < 1e-12
    assert np.abs(sh_real(l, -v) - (-1) ** l * sh_real(l, v)).max() < 1e-13


@pytest.mark.parametrize("l", range(4))
def test_wigner_d_group_properties(l):
    rng = np.random.default_rng(30 + l)
    r1, r2 = random_rotation(rng), random_rotation(rng)
    d1 = wigner_D_real(l, *euler_angles(r1))
    d2 = wigner_D_real(l, *euler_angles(r2))
    d12 = wigner_D_real(l, *euler_angles(r1 @ r2))
    assert np.abs(d1 @ d1.T - np.eye(2 * l + 1)).max() < 1e-12
    assert np.abs(d12 - d1 @ d2).max() < 1e-12
    assert np.abs(wigner_D_real(l, 0.0, 0.0, 0.0) - np.eye(2 * l + 1)).max() < 1e-15
    if l == 1:
        # the l = 1 real representation is the rotation matrix itself in (y, z, x) order
        perm = [1, 2, 0]
        assert np.abs(d1 - r1[np.ix_(perm, perm)]).max() < 1e-12


@pytest.mark.parametrize("l", range(4))
def test_sh_gradient_complex_step_and_tangent(l):
    rng = np.random.default_rng(40 + l)
    v = rng.standard_normal((20, 3)) * 2.0
    g = sh_real_grad(l, v)
    for k in range(3):
        vc = v.astype(np.complex128)
        vc[:, k] += 1e-30j
        cs = sh_real(l, vc).imag / 1e-30
        assert np.abs(cs - g[..., k]).max() < 1e-12
    # harmonics depend on direction only: the gradient is orthogonal to v
    assert np.abs(np.einsum("emk,ek->em", g, v)).max() < 1e-11


def test_envelope_boundary_values():
    assert envelope(0.0) == 1.0
    assert abs(envelope(1.0 - 1e-12)) < 1e-9
    assert envelope(1.0) == 0.0 and envelope(1.5) == 0.0
    # u'(1) = u''(1) = 0 and u'(t) matches finite differences
    h = 1e-6
    for t in (0.1, 0.5, 0.9):
        fd = (envelope(t + h) - envelope(t - h)) / (2 * h)
        assert abs(fd - envelope_deriv(t)) < 1e-8
    assert abs(envelope_deriv(1.0 - 1e-12)) < 1e-9
    # u' has a double root at t = 1 (so u''(1) = 0): u'(1 - e) / e^2 -> -p(p+1)(p+2)/2
    for eps in (1e-3, 1e-4, 1e-5):
        assert abs(envelope_deriv(1.0 - eps) / eps ** 2 + 168.0) < 168.0 * 6 * eps


def test_bessel_limits_and_derivatives():
    rc = 5.0
    # d -> 0 limit: (2/rc)(n pi / rc)
    b0 = bessel(np.array([1e-8]), 8, rc)[0]
    assert np.allclose(b0, 2.0 / rc * np.arange(1, 9) * np.pi / rc, rtol=1e-10)
    d = np.linspace(0.5, 4.9, 9)
    for fn, dfn in ((bessel, bessel_deriv), (radial, radial_deriv)):
        dc = d.astype(np.complex128) + 1e-30j
        cs = fn(dc, 8, rc).imag / 1e-30
        assert np.abs(cs - dfn(d, 8, rc)).max() < 1e-12
    assert np.all(radial(np.array([rc, rc + 1.0]), 8, rc) == 0.0)
