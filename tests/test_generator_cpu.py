"""The device code generator's inputs against the oracle, on the CPU.

The generator (product side) takes its Clebsch-Gordan values from sympy and its harmonic
polynomials from a fit to scipy's spherical harmonics; the oracle derives both from closed forms
(Racah's formula, solid harmonics). The two share no code; agreement here pins every coefficient
that the generated kernels carry as an immediate, without a GPU.
"""
import importlib.util
import os

import numpy as np
import pytest

from oracle.cg import cg_real
from oracle.sh import sh_real

_GEN = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "equivariant_mlip_tensor_edge_b200", "csrc", "gen_paths.py")


@pytest.fixture(scope="module")
def gen():
    spec = importlib.util.spec_from_file_location("gen_paths", _GEN)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_generator_couplings_equal_the_oracle_for_every_triple(gen):
    """All 65 couplings up to rank 4, even and odd l1 + l2 + l3, including the odd-sum sign."""
    tri = gen.gen_triples()
    assert len(tri) == 65
    for l1, l2, l3 in tri:
        a = gen.real_cg_any(l1, l2, l3)
        b = cg_real(l1, l2, l3)
        assert np.abs(a - b).max() < 1e-12, (l1, l2, l3)
    # the uniform kernels' path tables use the even couplings only
    for lmax in (1, 2, 3):
        for p in gen.paths_for(lmax):
            assert sum(p) % 2 == 0
            assert np.abs(gen.real_cg(*p) - cg_real(*p)).max() < 1e-12


@pytest.mark.parametrize("l", range(5))
def test_generator_harmonic_polynomials_equal_the_oracle(gen, l):
    rng = np.random.default_rng(l)
    v = rng.standard_normal((50, 3))
    v /= np.linalg.norm(v, axis=1, keepdims=True)
    coef = gen.sh_polynomials(l) if l > 0 else np.ones((1, 1))
    mons = gen.monomials(l)
    a = np.stack([v[:, 0] ** p * v[:, 1] ** q * v[:, 2] ** s for p, q, s in mons], axis=1)
    ours = a @ coef.T
    ref = sh_real(l, v)
    assert np.abs(ours - ref).max() < 1e-10


def test_generated_header_is_current(gen):
    """The committed header is what the generator writes now (no stale device code)."""
    path = os.path.join(os.path.dirname(_GEN), "generated", "etp_paths.h")
    with open(path) as f:
        assert f.read() == gen.generate()
