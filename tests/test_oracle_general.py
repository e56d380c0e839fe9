"""Pins for the oracle's general irreps: per-block multiplicities, paths with l1 + l2 + l3 odd
(real antisymmetric couplings) and rank 4 (CPU only)."""
import numpy as np
import pytest

import workloads
from oracle.cg import cg_real
from oracle.conv import ConvSpec, conv_forward, conv_vjp, conv_vjp_weights, flop_counts
from oracle.graph import csr, neighbors
from oracle.sh import sh_real
from oracle.wigner import euler_angles, random_rotation, wigner_D_real

# mixed multiplicities, both parities of l = 1 and 2, rank up to 4
MIXED = "4x0e+3x1o+3x1e+4x2e+2x2o+3x3o+4x4e"


def _triples(lmax):
    return [(a, b, c) for a in range(lmax + 1) for b in range(lmax + 1)
            for c in range(abs(a - b), min(lmax, a + b) + 1)]


@pytest.fixture(scope="module")
def graph():
    wl = workloads.make("tiny")
    nb = neighbors(wl.pos, wl.cell, wl.pbc, wl.r_cut)
    row_ptr, _, _ = csr(nb["receiver"], nb["sender"], wl.n_nodes)
    return dict(wl=wl, nb=nb, row_ptr=row_ptr)


def _setup(graph, irreps_in, sh_lmax, irreps_out, seed):
    spec = ConvSpec(irreps_in, sh_lmax, irreps_out, 8, float(graph["wl"].r_cut))
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((graph["wl"].n_nodes, spec.dim_in))
    W = rng.standard_normal((8, spec.weight_numel))
    g = rng.standard_normal((graph["wl"].n_nodes, spec.dim_out))
    return spec, x, W, g


def _block_rotation(blocks, a, b, c):
    dim = sum(m * (2 * l + 1) for m, l, _ in blocks)
    rot = np.zeros((dim, dim))
    off = 0
    for m, l, _ in blocks:
        d = wigner_D_real(l, a, b, c)
        for u in range(m):
            idx = off + np.arange(2 * l + 1) * m + u
            rot[np.ix_(idx, idx)] = d
        off += m * (2 * l + 1)
    return rot


# ----------------------------------------------------------------- couplings

def test_odd_coupling_1x1_to_1_is_the_cross_product():
    """For 1 x 1 -> 1 the real coupling is the cross product: with the l = 1 components ordered
    as the harmonics order them (m = -1, 0, 1 <-> y, z, x, read off Y_1 itself), it is
    epsilon / sqrt(2) up to an overall sign."""
    rng = np.random.default_rng(0)
    n = rng.standard_normal(3)
    n /= np.linalg.norm(n)
    y1 = sh_real(1, n[None, :])[0] / np.sqrt(3.0)
    order = [int(np.argmin(np.abs(np.abs(n) - abs(v)))) for v in y1]   # Cartesian axis of each m
    assert sorted(order) == [0, 1, 2]
    T = cg_real(1, 1, 1)
    eps = np.zeros((3, 3, 3))
    eps[0, 1, 2] = eps[1, 2, 0] = eps[2, 0, 1] = 1.0
    eps[0, 2, 1] = eps[2, 1, 0] = eps[1, 0, 2] = -1.0
    ref = eps[np.ix_(order, order, order)] / np.sqrt(2.0)
    sign = np.sign(T[0, 1, 2] / ref[0, 1, 2])
    assert np.abs(T - sign * ref).max() < 1e-14
    # antisymmetric in the two inputs
    assert np.abs(T + T.transpose(1, 0, 2)).max() < 1e-14


@pytest.mark.parametrize("l1,l2,l3", _triples(4))
def test_real_coupling_equivariant_and_orthonormal(l1, l2, l3):
    """Every real coupling up to rank 4, even and odd l1 + l2 + l3: rotating both inputs rotates
    the output (real Wigner matrices), and sum_{m1,m2} C[m1,m2,m3] C[m1,m2,m3'] = delta."""
    T = cg_real(l1, l2, l3)
    rng = np.random.default_rng(100 * l1 + 10 * l2 + l3)
    ang = euler_angles(random_rotation(rng))
    d1, d2, d3 = (wigner_D_real(l, *ang) for l in (l1, l2, l3))
    x, y = rng.standard_normal(2 * l1 + 1), rng.standard_normal(2 * l2 + 1)
    z = np.einsum("abc,a,b->c", T, x, y)
    zr = np.einsum("abc,a,b->c", T, d1 @ x, d2 @ y)
    assert np.abs(zr - d3 @ z).max() < 1e-12 * max(1.0, np.abs(z).max())
    gram = np.einsum("abc,abd->cd", T, T)
    assert np.abs(gram - np.eye(2 * l3 + 1)).max() < 1e-12


# ----------------------------------------------------------------- path set

def test_paths_pair_equal_multiplicities_and_parity():
    spec = ConvSpec("4x0e+2x1o", 1, "4x0e+3x1o", 8, 5.0)
    assert spec.paths == [(0, 0, 0)]           # 0e->1o (4 vs 3), 1o->1o (2 vs 3), 1o->0e (2 vs 4) dropped
    assert spec.weight_numel == 4 and spec.channels is None
    spec = ConvSpec(MIXED, 4, MIXED, 8, 5.0)
    for p, (bi, l2, bo) in enumerate(spec.paths):
        m1, l1, p1 = spec.blocks_in[bi]
        m3, l3, p3 = spec.blocks_out[bo]
        assert m1 == m3 == spec.path_mul[p] and abs(l1 - l2) <= l3 <= l1 + l2 and p1 * (-1) ** l2 == p3
    odd = [p for p in range(len(spec.paths)) if sum(spec.path_ls(p)) % 2]
    assert len(odd) > 0
    assert spec.woff == list(np.cumsum([0] + spec.path_mul)[:-1])
    fc = flop_counts(spec)
    assert fc["fwd_tp"] == sum(2 * (np.count_nonzero(cg_real(*spec.path_ls(p))) + 2 * spec.path_ls(p)[2] + 1)
                               * spec.path_mul[p] for p in range(len(spec.paths)))


# ----------------------------------------------------------------- forward

@pytest.mark.parametrize("irreps,sh_lmax", [(MIXED, 4), ("3x0e+3x1o+3x1e+3x2e+3x2o", 2),
                                            ("5x0e+4x1o+3x2e+2x3o", 3)])
def test_general_forward_rotation_and_inversion(graph, irreps, sh_lmax):
    spec, x, W, _ = _setup(graph, irreps, sh_lmax, irreps, 1)
    nb, rp = graph["nb"], graph["row_ptr"]
    vec = nb["edge_vec"].astype(np.float64)
    out = conv_forward(spec, rp, nb["sender"], vec, x, W)
    rng = np.random.default_rng(2)
    rot = random_rotation(rng)
    ang = euler_angles(rot)
    din, dout = _block_rotation(spec.blocks_in, *ang), _block_rotation(spec.blocks_out, *ang)
    out_r = conv_forward(spec, rp, nb["sender"], vec @ rot.T, x @ din.T, W)
    assert np.abs(out_r - out @ dout.T).max() < 1e-11 * max(1.0, np.abs(out).max())
    # inversion: each block carries its own parity; the harmonics carry (-1)^l2
    par_in = np.concatenate([np.full(m * (2 * l + 1), float(p)) for m, l, p in spec.blocks_in])
    par_out = np.concatenate([np.full(m * (2 * l + 1), float(p)) for m, l, p in spec.blocks_out])
    out_p = conv_forward(spec, rp, nb["sender"], -vec, x * par_in, W)
    assert np.abs(out_p - out * par_out).max() < 1e-12 * max(1.0, np.abs(out).max())


def test_general_single_path_isolation(graph):
    """Zeroing every weight column but path p's leaves output only in p's output block, and the
    single-path outputs add up to the full output: each path reads its own columns of W."""
    spec, x, W, _ = _setup(graph, MIXED, 4, MIXED, 3)
    nb, rp = graph["nb"], graph["row_ptr"]
    full = conv_forward(spec, rp, nb["sender"], nb["edge_vec"], x, W)
    acc = np.zeros_like(full)
    for p, (bi, l2, bo) in enumerate(spec.paths):
        Wp = np.zeros_like(W)
        Wp[:, spec.w_slice(p)] = W[:, spec.w_slice(p)]
        o = conv_forward(spec, rp, nb["sender"], nb["edge_vec"], x, Wp)
        outside = np.ones(spec.dim_out, dtype=bool)
        outside[spec.out_slice(bo)] = False
        assert np.abs(o[:, outside]).max() == 0.0
        assert np.abs(o[:, spec.out_slice(bo)]).max() > 0.0
        acc += o
    assert np.abs(acc - full).max() < 1e-12 * max(1.0, np.abs(full).max())


def test_general_uniform_case_keeps_the_uniform_layout(graph):
    """With one multiplicity C the flat weight layout is [n_basis, n_paths, C]."""
    spec, x, W, _ = _setup(graph, "4x0e+4x1o+4x1e+4x2e", 2, "4x0e+4x1o+4x1e+4x2e", 4)
    nb, rp = graph["nb"], graph["row_ptr"]
    a = conv_forward(spec, rp, nb["sender"], nb["edge_vec"], x, W)
    b = conv_forward(spec, rp, nb["sender"], nb["edge_vec"], x, W.reshape(8, len(spec.paths), 4))
    assert np.array_equal(a, b)


# ----------------------------------------------------------------- VJP

def test_general_vjp_complex_step_and_adjoint(graph):
    spec, x, W, g = _setup(graph, MIXED, 4, MIXED, 5)
    nb, rp = graph["nb"], graph["row_ptr"]
    vec = nb["edge_vec"].astype(np.float64)

    def loss(xx, vv, ww=W):
        return (conv_forward(spec, rp, nb["sender"], vv, xx, ww) * g).sum()

    gx, gv = conv_vjp(spec, rp, nb["sender"], vec, x, W, g)
    rng = np.random.default_rng(6)
    for _ in range(6):
        e, k = rng.integers(len(vec)), rng.integers(3)
        vc = vec.astype(np.complex128)
        vc[e, k] += 1e-30j
        cs = loss(x, vc).imag / 1e-30
        assert abs(cs - gv[e, k]) < 1e-11 * max(1.0, abs(cs))
    # the loss is linear in x and in W: directional differences are exact
    dx = rng.standard_normal(x.shape)
    assert abs(loss(x + dx, vec) - loss(x, vec) - (gx * dx).sum()) < 1e-9 * max(1.0, abs(loss(x, vec)))
    dW = rng.standard_normal(W.shape)
    gW = conv_vjp_weights(spec, rp, nb["sender"], vec, x, g)
    assert gW.shape == W.shape
    assert abs(loss(x, vec, W + dW) - loss(x, vec) - (gW * dW).sum()) < 1e-9 * max(1.0, abs(loss(x, vec)))
