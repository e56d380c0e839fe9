"""Pins for the oracle's Clebsch-Gordan coefficients (CPU only)."""
import os
from math import sqrt

import numpy as np
import pytest
from sympy import N as sym_n
from sympy.physics.wigner import clebsch_gordan

from oracle.cg import cg_complex, cg_real, real_basis
from oracle.wigner import euler_angles, random_rotation, wigner_D_real

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _triples(lmax, even_only=True):
    out = []
    for l1 in range(lmax + 1):
        for l2 in range(lmax + 1):
            for l3 in range(abs(l1 - l2), min(l1 + l2, lmax) + 1):
                if not even_only or (l1 + l2 + l3) % 2 == 0:
                    out.append((l1, l2, l3))
    return out


def test_racah_matches_sympy_library():
    # sympy's clebsch_gordan is an independent implementation (exact symbolic).
    for l1, l2, l3 in _triples(3, even_only=False) + [(4, 5, 3), (5, 5, 6)]:
        for m1 in range(-l1, l1 + 1):
            for m2 in range(-l2, l2 + 1):
                m3 = m1 + m2
                if abs(m3) > l3:
                    continue
                ref = float(sym_n(clebsch_gordan(l1, l2, l3, m1, m2, m3), 20))
                assert abs(cg_complex(l1, m1, l2, m2, l3, m3) - ref) < 1e-14


def test_textbook_values():
    for l1 in range(4):
        for l2 in range(4):
            assert abs(cg_complex(l1, l1, l2, l2, l1 + l2, l1 + l2) - 1.0) < 1e-15
    for m in (-1, 0, 1):
        assert abs(cg_complex(1, m, 1, -m, 0, 0) - (-1) ** (1 - m) / sqrt(3.0)) < 1e-15
    # selection rules
    assert cg_complex(1, 1, 1, 1, 2, 1) == 0.0
    assert cg_complex(1, 0, 1, 0, 3, 0) == 0.0


def test_real_basis_unitary():
    for l in range(5):
        q = real_basis(l)
        assert np.allclose(q @ q.conj().T, np.eye(2 * l + 1), atol=1e-15)


@pytest.mark.parametrize("l1,l2,l3", _triples(3))
def test_real_cg_orthonormal(l1, l2, l3):
    c = cg_real(l1, l2, l3)
    gram = np.einsum("abc,abd->cd", c, c)
    assert np.allclose(gram, np.eye(2 * l3 + 1), atol=1e-14)


@pytest.mark.parametrize("l1,l2,l3", _triples(3))
def test_real_cg_equivariant(l1, l2, l3):
    rng = np.random.default_rng(100 * l1 + 10 * l2 + l3)
    c = cg_real(l1, l2, l3)
    for _ in range(3):
        a, b, g = euler_angles(random_rotation(rng))
        d1, d2, d3 = (wigner_D_real(l, a, b, g) for l in (l1, l2, l3))
        lhs = np.einsum("abc,ai,bj->ijc", c, d1, d2)
        rhs = np.einsum("ijk,ck->ijc", c, d3)
        assert np.abs(lhs - rhs).max() < 1e-13


def test_table_c1_operation_counts():
    """FlashCart Table C1: couplings and sparse-CG op counts for max rank 3, 4, 5.

    Reading: couplings are (l1 <= l2, l3) with the triangle rule and l1+l2+l3
    even; a sparse real-CG coupling costs 3 ops per nonzero (two multiplies,
    one add) minus one add per output component and minus one multiply for the
    unit (0,0,0) coefficient: ops = 3 nnz - sum (2 l3 + 1) - 1.
    """
    rows = [list(map(int, ln.split())) for ln in open(os.path.join(GOLDEN, "table_c1.txt"))
            if ln.strip() and not ln.startswith("#")]
    for lmax, n_couplings, ops in rows:
        cps = [(a, b, c) for a in range(lmax + 1) for b in range(a, lmax + 1) for c in range(lmax + 1)
               if abs(a - b) <= c <= a + b and (a + b + c) % 2 == 0]
        assert len(cps) == n_couplings
        nnz = sum(int(np.count_nonzero(cg_real(*t))) for t in cps)
        assert 3 * nnz - sum(2 * c + 1 for _, _, c in cps) - 1 == ops


def test_cg_sparsity_is_exact_zeros():
    # entries that vanish by selection rules must be exactly zero, not rounding noise
    for t in _triples(3):
        c = cg_real(*t)
        nz = c[c != 0]
        assert np.abs(nz).min() > 1e-3
