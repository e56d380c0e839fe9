"""Pins for the oracle's node-local product and product ladder (CPU only)."""
import numpy as np
import pytest

from oracle.cg import cg_real
from oracle.product import node_ladder, node_product, product_paths
from oracle.wigner import euler_angles, random_rotation, wigner_D_real


def _rot_features(lmax, c, a, b, g):
    dim = (lmax + 1) ** 2 * c
    rot = np.zeros((dim, dim))
    for l in range(lmax + 1):
        d = wigner_D_real(l, a, b, g)
        for u in range(c):
            idx = l * l * c + np.arange(2 * l + 1) * c + u
            rot[np.ix_(idx, idx)] = d
    return rot


def test_path_set_counts():
    # same path set as the edge convolution with in = SH = out = L: 4, 11, 23 paths
    assert [len(product_paths(L)) for L in (1, 2, 3)] == [4, 11, 23]


@pytest.mark.parametrize("lmax", [1, 2, 3])
def test_product_equivariance_and_parity(lmax):
    rng = np.random.default_rng(40 + lmax)
    c, n = 3, 5
    dim = (lmax + 1) ** 2 * c
    A, B = rng.standard_normal((n, dim)), rng.standard_normal((n, dim))
    W = rng.standard_normal((len(product_paths(lmax)), c))
    out = node_product(lmax, c, B, A, W)
    rot = _rot_features(lmax, c, *euler_angles(random_rotation(rng)))
    out_r = node_product(lmax, c, B @ rot.T, A @ rot.T, W)
    assert np.abs(out_r - out @ rot.T).max() < 1e-11 * np.abs(out).max()
    par = np.concatenate([np.full((2 * l + 1) * c, (-1.0) ** l) for l in range(lmax + 1)])
    out_p = node_product(lmax, c, B * par, A * par, W)
    assert np.abs(out_p - out * par).max() < 1e-12 * np.abs(out).max()


def test_product_single_path_brute_force():
    # one path at a time against explicit loops over m1, m2, m3 (channels independent)
    rng = np.random.default_rng(41)
    lmax, c, n = 2, 2, 3
    dim = 9 * c
    A, B = rng.standard_normal((n, dim)), rng.standard_normal((n, dim))
    paths = product_paths(lmax)
    for p, (l1, l2, l3) in enumerate(paths):
        W = np.zeros((len(paths), c))
        W[p] = rng.standard_normal(c)
        out = node_product(lmax, c, B, A, W)
        cg = cg_real(l1, l2, l3)
        ref = np.zeros_like(out)
        for i in range(n):
            for u in range(c):
                for m1 in range(2 * l1 + 1):
                    for m2 in range(2 * l2 + 1):
                        for m3 in range(2 * l3 + 1):
                            ref[i, (l3 * l3 + m3) * c + u] += (W[p, u] * cg[m1, m2, m3] *
                                                              B[i, (l1 * l1 + m1) * c + u] *
                                                              A[i, (l2 * l2 + m2) * c + u])
        assert np.abs(out - ref).max() < 1e-13


def test_scalar_path_is_the_elementwise_product():
    # the (0, 0, 0) path: P[0, u] = W[0, u] B[0, u] A[0, u]
    rng = np.random.default_rng(42)
    c, n = 4, 6
    A, B = rng.standard_normal((n, 4 * c)), rng.standard_normal((n, 4 * c))
    W = np.zeros((4, c))
    W[0] = rng.standard_normal(c)
    out = node_product(1, c, B, A, W)
    assert np.abs(out[:, :c] - W[0] * B[:, :c] * A[:, :c]).max() < 1e-14
    assert np.abs(out[:, c:]).max() == 0.0


def test_ladder_recursion():
    rng = np.random.default_rng(43)
    lmax, c, n = 2, 3, 4
    dim = 9 * c
    A = rng.standard_normal((n, dim))
    Ws = rng.standard_normal((3, len(product_paths(lmax)), c))
    assert np.array_equal(node_ladder(lmax, c, A, Ws[:0]), A)
    b2 = node_product(lmax, c, A, A, Ws[0])
    b3 = node_product(lmax, c, b2, A, Ws[1])
    b4 = node_product(lmax, c, b3, A, Ws[2])
    assert np.abs(node_ladder(lmax, c, A, Ws) - (A + b2 + b3 + b4)).max() < 1e-12 * np.abs(b4).max()
    # a ladder of order nu is a polynomial of degree nu in A: scaling A by s scales B_q by s^q
    s = 1.7
    lad = node_ladder(lmax, c, s * A, Ws[:1])
    assert np.abs(lad - (s * A + s * s * b2)).max() < 1e-12 * np.abs(lad).max()


# ---------------------------------------------------------------- the full ladder ("FlashCart",
# Fig. 3b dashed curves and Fig. E1 (b): per-rank matrices that mix paths and channels)

def _diagonal_full_step(lmax, c, w):
    """The full step whose rank-l3 matrix is W_l3[v, p' C + u] = delta_uv w[p, u]."""
    from oracle.product import paths_of_rank
    blocks = []
    for l3 in range(lmax + 1):
        ps = paths_of_rank(lmax, l3)
        m = np.zeros((c, len(ps) * c))
        for j, p in enumerate(ps):
            m[np.arange(c), j * c + np.arange(c)] = w[p]
        blocks.append(m.ravel())
    return np.concatenate(blocks)


@pytest.mark.parametrize("lmax", [1, 2, 3])
def test_full_step_with_channel_diagonal_weights_is_the_path_reduced_product(lmax):
    from oracle.product import node_product_full
    rng = np.random.default_rng(70 + lmax)
    c, n = 3, 4
    dim = (lmax + 1) ** 2 * c
    A, B = rng.standard_normal((n, dim)), rng.standard_normal((n, dim))
    w = rng.standard_normal((len(product_paths(lmax)), c))
    ref = node_product(lmax, c, B, A, w)
    got = node_product_full(lmax, c, B, A, _diagonal_full_step(lmax, c, w))
    assert np.abs(got - ref).max() < 1e-12 * np.abs(ref).max()


@pytest.mark.parametrize("lmax", [1, 2, 3])
def test_full_step_equivariance_and_parity(lmax):
    from oracle.product import full_step_sizes, node_product_full
    rng = np.random.default_rng(80 + lmax)
    c, n = 3, 5
    dim = (lmax + 1) ** 2 * c
    A, B = rng.standard_normal((n, dim)), rng.standard_normal((n, dim))
    w = rng.standard_normal(sum(full_step_sizes(lmax, c)))
    out = node_product_full(lmax, c, B, A, w)
    rot = _rot_features(lmax, c, *euler_angles(random_rotation(rng)))
    out_r = node_product_full(lmax, c, B @ rot.T, A @ rot.T, w)
    assert np.abs(out_r - out @ rot.T).max() < 1e-11 * np.abs(out).max()
    par = np.concatenate([np.full((2 * l + 1) * c, (-1.0) ** l) for l in range(lmax + 1)])
    out_p = node_product_full(lmax, c, B * par, A * par, w)
    assert np.abs(out_p - out * par).max() < 1e-12 * np.abs(out).max()


def test_full_step_brute_force():
    # every index by explicit loops: B'[l3 m3 v] = sum_{p of l3, u} W[v, p' C + u] sum_{m1 m2} C B A
    from oracle.product import full_step_sizes, node_product_full, paths_of_rank, split_full_step
    rng = np.random.default_rng(90)
    lmax, c, n = 2, 2, 2
    dim = 9 * c
    A, B = rng.standard_normal((n, dim)), rng.standard_normal((n, dim))
    w = rng.standard_normal(sum(full_step_sizes(lmax, c)))
    mats = split_full_step(lmax, c, w)
    paths = product_paths(lmax)
    ref = np.zeros((n, dim))
    for i in range(n):
        for l3 in range(lmax + 1):
            for j, p in enumerate(paths_of_rank(lmax, l3)):
                l1, l2, _ = paths[p]
                cg = cg_real(l1, l2, l3)
                for u in range(c):
                    for m1 in range(2 * l1 + 1):
                        for m2 in range(2 * l2 + 1):
                            for m3 in range(2 * l3 + 1):
                                t = cg[m1, m2, m3] * B[i, (l1 * l1 + m1) * c + u] * A[i, (l2 * l2 + m2) * c + u]
                                for v in range(c):
                                    ref[i, (l3 * l3 + m3) * c + v] += mats[l3][v, j * c + u] * t
    assert np.abs(node_product_full(lmax, c, B, A, w) - ref).max() < 1e-13


def test_full_ladder_recursion():
    from oracle.product import full_step_sizes, node_ladder_full, node_product_full
    rng = np.random.default_rng(91)
    lmax, c, n = 2, 3, 4
    A = rng.standard_normal((n, 9 * c))
    Ws = [rng.standard_normal(sum(full_step_sizes(lmax, c))) for _ in range(2)]
    assert np.array_equal(node_ladder_full(lmax, c, A, []), A)
    b2 = node_product_full(lmax, c, A, A, Ws[0])
    b3 = node_product_full(lmax, c, b2, A, Ws[1])
    assert np.abs(node_ladder_full(lmax, c, A, Ws) - (A + b2 + b3)).max() < 1e-12 * np.abs(b3).max()
    # with channel-diagonal steps the full ladder is the path-reduced one
    wr = rng.standard_normal((2, len(product_paths(lmax)), c))
    full = node_ladder_full(lmax, c, A, [_diagonal_full_step(lmax, c, x) for x in wr])
    red = node_ladder(lmax, c, A, wr)
    assert np.abs(full - red).max() < 1e-12 * np.abs(red).max()
