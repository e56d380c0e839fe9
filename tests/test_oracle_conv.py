"""Pins for the oracle's neighbour list, CSR, forward convolution and VJP (CPU only)."""
import numpy as np
import pytest
from scipy.spatial import cKDTree

import workloads
from oracle.cg import cg_real
from oracle.conv import ConvSpec, conv_forward, conv_vjp, conv_vjp_weights, flop_counts, parse_irreps
from oracle.graph import csr, forces_from_edge_grads, neighbors
from oracle.radial import radial
from oracle.wigner import euler_angles, random_rotation, wigner_D_real


@pytest.fixture(scope="module")
def tiny():
    wl = workloads.make("tiny")
    nb = neighbors(wl.pos, wl.cell, wl.pbc, wl.r_cut)
    row_ptr, t_row_ptr, t_perm = csr(nb["receiver"], nb["sender"], wl.n_nodes)
    spec = ConvSpec(wl.irreps, wl.lmax, wl.irreps, wl.n_basis, float(wl.r_cut))
    x = wl.features().astype(np.float64)
    w = wl.weights(len(spec.paths)).astype(np.float64)
    g = wl.cotangent().astype(np.float64)
    return dict(wl=wl, nb=nb, row_ptr=row_ptr, spec=spec, x=x, W=w, g=g)


# ----------------------------------------------------------------- graph

def _kdtree_pairs(pos, box, r_cut):
    tree = cKDTree(pos, boxsize=box)
    pairs = tree.query_pairs(r_cut, output_type="ndarray")
    out = set()
    for i, j in pairs:
        out.add((int(i), int(j)))
        out.add((int(j), int(i)))
    return out


@pytest.mark.parametrize("name", ["tiny", "diamond1k"])
def test_neighbors_match_kdtree(name):
    wl = workloads.make(name)
    nb = neighbors(wl.pos, wl.cell, wl.pbc, wl.r_cut)
    pos = wl.pos.astype(np.float64)
    box = None if wl.cell is None else np.diag(wl.cell)
    if box is not None:
        pos = np.mod(pos, box)
    ref = _kdtree_pairs(pos, box, float(wl.r_cut))
    got = set(zip(nb["receiver"].tolist(), nb["sender"].tolist()))
    # every periodic cell here is wider than 2 r_cut: at most one image per pair
    assert len(got) == len(nb["receiver"])
    d = np.linalg.norm(nb["edge_vec"].astype(np.float64), axis=1)
    assert np.all(d < float(wl.r_cut) + 1e-6)
    assert got == ref


def test_perfect_diamond_shell_count():
    # a = 3.567 A, r < 5 A: shells 4 + 12 + 12 + 6 + 12 + 24 + 16 = 86 (next shell 5.044 A)
    a, n = 3.567, 3
    basis = np.array([[0, 0, 0], [0, .5, .5], [.5, 0, .5], [.5, .5, 0],
                      [.25, .25, .25], [.25, .75, .75], [.75, .25, .75], [.75, .75, .25]])
    grid = np.stack(np.meshgrid(*[np.arange(n)] * 3, indexing="ij"), -1).reshape(-1, 3)
    pos = ((grid[:, None, :] + basis[None]).reshape(-1, 3) * a).astype(np.float32)
    nb = neighbors(pos, np.eye(3) * n * a, (True, True, True), np.float32(5.0), receivers=[0, 5, 100])
    counts = np.bincount(nb["receiver"], minlength=101)
    assert counts[0] == counts[5] == counts[100] == 86


def test_canonical_order_and_csr(tiny):
    nb = tiny["nb"]
    key = np.stack([nb["receiver"], nb["sender"], nb["shift"][:, 0], nb["shift"][:, 1], nb["shift"][:, 2]], 1)
    assert all(tuple(key[k]) < tuple(key[k + 1]) for k in range(len(key) - 1))
    row_ptr, t_row_ptr, t_perm = csr(nb["receiver"], nb["sender"], tiny["wl"].n_nodes)
    assert row_ptr[0] == 0 and row_ptr[-1] == len(key) and np.all(np.diff(row_ptr) >= 0)
    assert sorted(t_perm.tolist()) == list(range(len(key)))
    tk = key[t_perm][:, [1, 0, 2, 3, 4]]
    assert all(tuple(tk[k]) < tuple(tk[k + 1]) for k in range(len(tk) - 1))
    assert np.array_equal(np.diff(t_row_ptr), np.bincount(nb["sender"], minlength=tiny["wl"].n_nodes))
    # the edge vector is sender - receiver (non-periodic case)
    pos = tiny["wl"].pos.astype(np.float64)
    ref = (pos[nb["sender"]] - pos[nb["receiver"]]).astype(np.float32)
    assert np.array_equal(ref, nb["edge_vec"])


# ----------------------------------------------------------------- paths

def test_irreps_and_path_enumeration():
    assert parse_irreps("64x0e+64x1o + 64x2e") == [(64, 0, 1), (64, 1, -1), (64, 2, 1)]
    assert parse_irreps("1o") == [(1, 1, -1)]
    with pytest.raises(ValueError):
        parse_irreps("64y0e")
    counts = {}
    for lmax in (1, 2, 3):
        irr = "+".join(f"4x{l}{'eo'[l % 2]}" for l in range(lmax + 1))
        spec = ConvSpec(irr, lmax, irr, 8, 5.0)
        fc = flop_counts(spec)
        counts[lmax] = (len(spec.paths), fc["nnz"], fc["sum_2l3p1"])
        for p in range(len(spec.paths)):
            l1, l2, l3 = spec.path_ls(p)
            assert abs(l1 - l2) <= l3 <= l1 + l2 and (l1 + l2 + l3) % 2 == 0
        assert spec.paths == sorted(spec.paths)
    # path counts, real-CG nonzeros and output components over the conv path set
    assert counts == {1: (4, 10, 8), 2: (11, 83, 35), 3: (23, 353, 99)}


# ----------------------------------------------------------------- forward

def test_direction_convention_closed_form():
    # two atoms on the z axis: edge (0 <- 1) has r = +z, Y_1(z) = sqrt(3) (y, z, x) = (0, sqrt(3), 0)
    spec = ConvSpec("1x0e+1x1o", 1, "1x0e+1x1o", 8, 4.0)
    row_ptr = np.array([0, 1, 2])
    sender = np.array([1, 0])
    vec = np.array([[0.0, 0.0, 1.5], [0.0, 0.0, -1.5]])
    x = np.zeros((2, 4))
    x[1, 0] = 2.0          # scalar feature on atom 1
    w = np.zeros((8, len(spec.paths), 1))
    p011 = spec.paths.index((0, 1, 1))
    w[:, p011, 0] = 1.0
    out = conv_forward(spec, row_ptr, sender, vec, x, w)
    wsum = radial(np.array([1.5]), 8, np.float64(np.float32(4.0)))[0].sum()
    assert np.allclose(out[0], [0.0, 0.0, 2.0 * wsum * np.sqrt(3.0), 0.0], atol=1e-14)
    assert np.allclose(out[1], 0.0)


def test_single_path_isolation(tiny):
    spec, x = tiny["spec"], tiny["x"]
    c = spec.channels
    for p, (bi, l2, bo) in enumerate(spec.paths):
        w = np.zeros_like(tiny["W"])
        w[3, p, 5] = 1.0
        out = conv_forward(spec, tiny["row_ptr"], tiny["nb"]["sender"], tiny["nb"]["edge_vec"], x, w)
        mask = np.zeros(spec.dim_out, bool)
        blk = np.arange(spec.dim_out)[spec.out_slice(bo)].reshape(-1, c)
        mask[blk[:, 5]] = True
        assert np.abs(out[:, ~mask]).max() == 0.0
        assert np.abs(out[:, mask]).max() > 0.0


def test_scalar_only_reduces_to_continuous_filter(tiny):
    # lmax = 0, 0e only: out[i,u] = sum_{j in N(i)} (sum_b R_b(d_ij) W[b,u]) x[j,u], brute force loops
    spec = ConvSpec("8x0e", 0, "8x0e", 8, float(tiny["wl"].r_cut))
    nb = tiny["nb"]
    rng = np.random.default_rng(7)
    x = rng.standard_normal((tiny["wl"].n_nodes, 8))
    w = rng.standard_normal((8, 1, 8))
    out = conv_forward(spec, tiny["row_ptr"], nb["sender"], nb["edge_vec"], x, w)
    ref = np.zeros_like(out)
    rc = np.float64(np.float32(spec.r_cut))
    for e in range(len(nb["sender"])):
        i, j = nb["receiver"][e], nb["sender"][e]
        d = float(np.linalg.norm(nb["edge_vec"][e].astype(np.float64)))
        rb = radial(np.array([d]), 8, rc)[0]
        for u in range(8):
            ref[i, u] += sum(rb[b] * w[b, 0, u] for b in range(8)) * x[j, u]
    assert np.abs(out - ref).max() < 1e-12


def _block_rotation(spec, blocks, a, b, g):
    dim = sum(m * (2 * l + 1) for m, l, _ in blocks)
    rot = np.zeros((dim, dim))
    off = 0
    for m, l, _ in blocks:
        d = wigner_D_real(l, a, b, g)
        for u in range(m):
            idx = off + np.arange(2 * l + 1) * m + u
            rot[np.ix_(idx, idx)] = d
        off += m * (2 * l + 1)
    return rot


@pytest.mark.parametrize("lmax", [1, 2, 3])
def test_forward_equivariance(tiny, lmax):
    irr = "+".join(f"3x{l}{'eo'[l % 2]}" for l in range(lmax + 1))
    spec = ConvSpec(irr, lmax, irr, 8, float(tiny["wl"].r_cut))
    nb = tiny["nb"]
    rng = np.random.default_rng(lmax)
    x = rng.standard_normal((tiny["wl"].n_nodes, spec.dim_in))
    w = rng.standard_normal((8, len(spec.paths), 3))
    vec = nb["edge_vec"].astype(np.float64)
    out = conv_forward(spec, tiny["row_ptr"], nb["sender"], vec, x, w)
    rot = random_rotation(rng)
    ang = euler_angles(rot)
    din = _block_rotation(spec, spec.blocks_in, *ang)
    dout = _block_rotation(spec, spec.blocks_out, *ang)
    out_r = conv_forward(spec, tiny["row_ptr"], nb["sender"], vec @ rot.T, x @ din.T, w)
    assert np.abs(out_r - out @ dout.T).max() < 1e-11 * max(1.0, np.abs(out).max())
    # inversion: odd harmonics flip, so with x -> parity-transformed x the output transforms by parity
    par_in = np.concatenate([np.full(m * (2 * l + 1), (-1.0) ** l) for m, l, _ in spec.blocks_in])
    par_out = np.concatenate([np.full(m * (2 * l + 1), (-1.0) ** l) for m, l, _ in spec.blocks_out])
    out_p = conv_forward(spec, tiny["row_ptr"], nb["sender"], -vec, x * par_in, w)
    assert np.abs(out_p - out * par_out).max() < 1e-12 * max(1.0, np.abs(out).max())


def test_forward_linearity(tiny):
    spec, nb = tiny["spec"], tiny["nb"]
    args = (spec, tiny["row_ptr"], nb["sender"], nb["edge_vec"])
    x, w = tiny["x"], tiny["W"]
    rng = np.random.default_rng(3)
    x2, w2 = rng.standard_normal(x.shape), rng.standard_normal(w.shape)
    f = lambda xx, ww: conv_forward(*args, xx, ww)
    assert np.allclose(f(2.0 * x - x2, w), 2.0 * f(x, w) - f(x2, w), atol=1e-12)
    assert np.allclose(f(x, 3.0 * w + w2), 3.0 * f(x, w) + f(x, w2), atol=1e-12)


def test_forward_permutation_equivariance(tiny):
    wl, spec = tiny["wl"], tiny["spec"]
    perm = np.random.default_rng(5).permutation(wl.n_nodes)
    nb2 = neighbors(wl.pos[perm], wl.cell, wl.pbc, wl.r_cut)
    rp2, _, _ = csr(nb2["receiver"], nb2["sender"], wl.n_nodes)
    out = conv_forward(spec, tiny["row_ptr"], tiny["nb"]["sender"], tiny["nb"]["edge_vec"], tiny["x"], tiny["W"])
    out2 = conv_forward(spec, rp2, nb2["sender"], nb2["edge_vec"], tiny["x"][perm], tiny["W"])
    assert np.abs(out2 - out[perm]).max() < 1e-12


def test_receiver_subset_matches_full(tiny):
    spec, nb = tiny["spec"], tiny["nb"]
    full = conv_forward(spec, tiny["row_ptr"], nb["sender"], nb["edge_vec"], tiny["x"], tiny["W"])
    sub = [0, 7, 19, 31]
    part = conv_forward(spec, tiny["row_ptr"], nb["sender"], nb["edge_vec"], tiny["x"], tiny["W"], receivers=sub)
    assert np.abs(part - full[sub]).max() == 0.0


# ----------------------------------------------------------------- backward

def _loss(tiny, x, vec):
    spec, nb = tiny["spec"], tiny["nb"]
    return (conv_forward(spec, tiny["row_ptr"], nb["sender"], vec, x, tiny["W"]) * tiny["g"]).sum()


def test_vjp_against_finite_differences_and_complex_step(tiny):
    spec, nb = tiny["spec"], tiny["nb"]
    gx, gv = conv_vjp(spec, tiny["row_ptr"], nb["sender"], nb["edge_vec"], tiny["x"], tiny["W"], tiny["g"])
    x = tiny["x"]
    vec = nb["edge_vec"].astype(np.float64)
    rng = np.random.default_rng(11)
    h = 1e-6
    for _ in range(6):
        e, k = rng.integers(len(vec)), rng.integers(3)
        vp, vm = vec.copy(), vec.copy()
        vp[e, k] += h
        vm[e, k] -= h
        fd = (_loss(tiny, x, vp) - _loss(tiny, x, vm)) / (2 * h)
        vc = vec.astype(np.complex128)
        vc[e, k] += 1e-30j
        cs = _loss(tiny, x, vc).imag / 1e-30
        assert abs(cs - gv[e, k]) < 1e-12 * max(1.0, abs(cs))
        assert abs(fd - gv[e, k]) < 1e-6 * max(1.0, abs(fd))
        a, b = rng.integers(x.shape[0]), rng.integers(x.shape[1])
        xp, xm = x.copy(), x.copy()
        xp[a, b] += h
        xm[a, b] -= h
        fdx = (_loss(tiny, xp, vec) - _loss(tiny, xm, vec)) / (2 * h)
        assert abs(fdx - gx[a, b]) < 1e-6 * max(1.0, abs(fdx))
    # grad_x is exact: the loss is linear in x
    xc = x.astype(np.complex128)
    xc[3, 2] += 1e-30j
    assert abs(_loss(tiny, xc, vec).imag / 1e-30 - gx[3, 2]) < 1e-12


def test_path_mask_partitions_the_forward(tiny):
    # paths are independent terms: a mask and its complement add up to the unmasked output, a
    # single-path mask equals the forward with the other paths' weights zeroed, all-ones is a no-op
    spec, nb = tiny["spec"], tiny["nb"]
    n_e, n_p = len(nb["sender"]), len(spec.paths)
    rng = np.random.default_rng(14)
    mask = rng.integers(0, 1 << n_p, size=n_e)
    full = conv_forward(spec, tiny["row_ptr"], nb["sender"], nb["edge_vec"], tiny["x"], tiny["W"])
    a = conv_forward(spec, tiny["row_ptr"], nb["sender"], nb["edge_vec"], tiny["x"], tiny["W"], path_mask=mask)
    b = conv_forward(spec, tiny["row_ptr"], nb["sender"], nb["edge_vec"], tiny["x"], tiny["W"],
                     path_mask=((1 << n_p) - 1) ^ mask)
    assert np.abs(a + b - full).max() < 1e-12 * np.abs(full).max()
    ones = conv_forward(spec, tiny["row_ptr"], nb["sender"], nb["edge_vec"], tiny["x"], tiny["W"],
                        path_mask=np.full(n_e, (1 << n_p) - 1))
    assert np.array_equal(ones, full)
    p = 2
    only = conv_forward(spec, tiny["row_ptr"], nb["sender"], nb["edge_vec"], tiny["x"], tiny["W"],
                        path_mask=np.full(n_e, 1 << p))
    w2 = np.zeros_like(tiny["W"])
    w2[:, p, :] = tiny["W"][:, p, :]
    ref = conv_forward(spec, tiny["row_ptr"], nb["sender"], nb["edge_vec"], tiny["x"], w2)
    assert np.abs(only - ref).max() < 1e-13 * max(1.0, np.abs(ref).max())


def test_masked_vjp_against_finite_differences(tiny):
    spec, nb = tiny["spec"], tiny["nb"]
    n_e, n_p = len(nb["sender"]), len(spec.paths)
    mask = np.random.default_rng(15).integers(0, 1 << n_p, size=n_e)
    gx, gv = conv_vjp(spec, tiny["row_ptr"], nb["sender"], nb["edge_vec"], tiny["x"], tiny["W"], tiny["g"],
                      path_mask=mask)
    vec = nb["edge_vec"].astype(np.float64)

    def loss(v):
        out = conv_forward(spec, tiny["row_ptr"], nb["sender"], v, tiny["x"], tiny["W"], path_mask=mask)
        return float((tiny["g"] * out).sum().real) if not np.iscomplexobj(out) else (tiny["g"] * out).sum()

    rng = np.random.default_rng(16)
    for _ in range(4):
        e, k = rng.integers(n_e), rng.integers(3)
        vc = vec.astype(np.complex128)
        vc[e, k] += 1e-30j
        cs = loss(vc).imag / 1e-30
        assert abs(cs - gv[e, k]) < 1e-12 * max(1.0, abs(cs))
    # grad_x: the loss is linear in x
    xc = tiny["x"].astype(np.complex128)
    xc[5, 3] += 1e-30j
    out = conv_forward(spec, tiny["row_ptr"], nb["sender"], vec, xc, tiny["W"], path_mask=mask)
    assert abs((tiny["g"] * out).sum().imag / 1e-30 - gx[5, 3]) < 1e-12


def test_weight_gradient_is_the_adjoint_of_the_forward(tiny):
    # the forward is linear in W: <dL/dW, V> = <g, F(x; W = V)> for every V, exactly
    spec, nb = tiny["spec"], tiny["nb"]
    dw = conv_vjp_weights(spec, tiny["row_ptr"], nb["sender"], nb["edge_vec"], tiny["x"], tiny["g"])
    assert dw.shape == (spec.n_basis, len(spec.paths), spec.channels)
    rng = np.random.default_rng(12)
    for _ in range(3):
        v = rng.standard_normal(dw.shape)
        out = conv_forward(spec, tiny["row_ptr"], nb["sender"], nb["edge_vec"], tiny["x"], v)
        lhs = float((dw * v).sum())
        rhs = float((tiny["g"] * out).sum())
        assert abs(lhs - rhs) < 1e-10 * max(1.0, abs(rhs))
    # a single nonzero entry of V picks out one entry of dW
    v = np.zeros(dw.shape)
    v[3, 2, 5] = 1.0
    out = conv_forward(spec, tiny["row_ptr"], nb["sender"], nb["edge_vec"], tiny["x"], v)
    assert abs(dw[3, 2, 5] - float((tiny["g"] * out).sum())) < 1e-12 * max(1.0, abs(dw[3, 2, 5]))


def test_weight_gradient_scalar_only_brute_force(tiny):
    # lmax = 0, 0e only: dL/dW[b,0,u] = sum_e R_b(d_e) g[recv,u] x[send,u], brute force loops
    spec = ConvSpec("8x0e", 0, "8x0e", 8, float(tiny["wl"].r_cut))
    nb = tiny["nb"]
    rng = np.random.default_rng(8)
    n = tiny["wl"].n_nodes
    x = rng.standard_normal((n, 8))
    g = rng.standard_normal((n, 8))
    dw = conv_vjp_weights(spec, tiny["row_ptr"], nb["sender"], nb["edge_vec"], x, g)
    ref = np.zeros((8, 1, 8))
    rc = np.float64(np.float32(spec.r_cut))
    for e in range(len(nb["sender"])):
        i, j = nb["receiver"][e], nb["sender"][e]
        d = float(np.linalg.norm(nb["edge_vec"][e].astype(np.float64)))
        rb = radial(np.array([d]), 8, rc)[0]
        for b in range(8):
            for u in range(8):
                ref[b, 0, u] += rb[b] * g[i, u] * x[j, u]
    assert np.abs(dw - ref).max() < 1e-12


def test_forces_sum_and_torque(tiny):
    spec, nb, wl = tiny["spec"], tiny["nb"], tiny["wl"]
    # rotation-invariant loss: L = <a, out_0e>  (scalar block only)
    rng = np.random.default_rng(2)
    g = np.zeros_like(tiny["g"])
    g[:, spec.out_slice(0)] = rng.standard_normal((wl.n_nodes, spec.channels))
    _, gv = conv_vjp(spec, tiny["row_ptr"], nb["sender"], nb["edge_vec"], tiny["x"], tiny["W"], g)
    f = forces_from_edge_grads(gv, nb["receiver"], nb["sender"], wl.n_nodes)
    assert np.abs(f.sum(0)).max() < 1e-12 * max(1.0, np.abs(f).max())
    # torque vanishes for a rotation-invariant loss with rotation-invariant (scalar-only) inputs
    xs = np.zeros_like(tiny["x"])
    xs[:, spec.in_slice(0)] = tiny["x"][:, spec.in_slice(0)]
    _, gv = conv_vjp(spec, tiny["row_ptr"], nb["sender"], nb["edge_vec"], xs, tiny["W"], g)
    # the loss depends on the edge vectors only, so its rotation invariance gives
    # sum_e r_e x dL/dr_e = 0 (the float32 edge vectors are the inputs here)
    torque = np.cross(nb["edge_vec"].astype(np.float64), gv).sum(0)
    assert np.abs(torque).max() < 1e-11 * max(1.0, np.abs(gv).max())


def test_flop_counts_formulae(tiny):
    fc = flop_counts(tiny["spec"])
    c = tiny["spec"].channels
    assert fc["fwd_tp"] == 2 * (10 + 8) * c
    assert fc["radial_proj"] == 2 * 8 * 4 * c
    nnz = sum(int(np.count_nonzero(cg_real(*tiny["spec"].path_ls(p)))) for p in range(4))
    assert fc["nnz"] == nnz


# ----------------------------------------------------------------- forces and periodic images

def _edges_from_positions(pos, nb, cell):
    """Edge vectors rebuilt from atom positions with the neighbour set held fixed:
    r_e = pos[sender] - pos[receiver] + S cell (float64)."""
    shift = nb["shift"].astype(np.float64)
    sv = shift @ (np.zeros((3, 3)) if cell is None else np.asarray(cell, dtype=np.float64))
    return pos[nb["sender"]] - pos[nb["receiver"]] + sv


def test_forces_are_minus_the_position_gradient(tiny):
    """F = -dL/dpos by central differences in the atom positions (neighbour set fixed), for
    L = <g, out>: pins the sign of forces_from_edge_grads and which end of an edge gets +g."""
    spec, nb, wl = tiny["spec"], tiny["nb"], tiny["wl"]
    pos = wl.pos.astype(np.float64)

    def loss(p):
        vec = _edges_from_positions(p, nb, wl.cell)
        return (conv_forward(spec, tiny["row_ptr"], nb["sender"], vec, tiny["x"], tiny["W"]) * tiny["g"]).sum()

    vec = _edges_from_positions(pos, nb, wl.cell)
    _, gv = conv_vjp(spec, tiny["row_ptr"], nb["sender"], vec, tiny["x"], tiny["W"], tiny["g"])
    f = forces_from_edge_grads(gv, nb["receiver"], nb["sender"], wl.n_nodes)
    h = 1e-6
    rng = np.random.default_rng(5)
    for _ in range(8):
        k, a = int(rng.integers(wl.n_nodes)), int(rng.integers(3))
        pp, pm = pos.copy(), pos.copy()
        pp[k, a] += h
        pm[k, a] -= h
        fd = (loss(pp) - loss(pm)) / (2 * h)
        assert abs(f[k, a] + fd) < 1e-6 * max(1.0, abs(fd)), (k, a, f[k, a], fd)
    # a flipped convention (receiver and sender swapped) gives -F and fails the check above
    assert np.abs(f).max() > 1e-3


def test_torque_of_the_forces_vanishes(tiny):
    """sum_i pos_i x F_i = 0 for a rotation-invariant loss of a non-periodic system: with
    scalar-only features, L = <a, out_0e> does not change when all positions rotate."""
    spec, nb, wl = tiny["spec"], tiny["nb"], tiny["wl"]
    assert wl.cell is None
    rng = np.random.default_rng(3)
    g = np.zeros_like(tiny["g"])
    g[:, spec.out_slice(0)] = rng.standard_normal((wl.n_nodes, spec.channels))
    xs = np.zeros_like(tiny["x"])
    xs[:, spec.in_slice(0)] = tiny["x"][:, spec.in_slice(0)]
    pos = wl.pos.astype(np.float64)
    vec = _edges_from_positions(pos, nb, None)
    _, gv = conv_vjp(spec, tiny["row_ptr"], nb["sender"], vec, xs, tiny["W"], g)
    f = forces_from_edge_grads(gv, nb["receiver"], nb["sender"], wl.n_nodes)
    assert np.abs(f.sum(0)).max() < 1e-12 * max(1.0, np.abs(f).max())
    torque = np.cross(pos, f).sum(0)
    assert np.abs(torque).max() < 1e-10 * max(1.0, np.abs(f).max() * np.abs(pos).max())
    # and it is a real check: with vector features the loss is not invariant and the torque is not 0
    _, gv2 = conv_vjp(spec, tiny["row_ptr"], nb["sender"], vec, tiny["x"], tiny["W"], tiny["g"])
    f2 = forces_from_edge_grads(gv2, nb["receiver"], nb["sender"], wl.n_nodes)
    assert np.abs(np.cross(pos, f2).sum(0)).max() > 1e-6


def _cell_case(case):
    """The periodic cells of the GPU image-scan tests (same seeds and shapes)."""
    if case == "orthorhombic_small":
        cell, n, seed, pbc = np.diag([7.1, 7.6, 8.3]), 40, 21, (True, True, True)
    elif case == "triclinic":
        cell, n, seed, pbc = [[11.0, 0.0, 0.0], [3.1, 10.5, 0.0], [-1.7, 2.2, 12.0]], 60, 22, (True, True, True)
    else:
        cell, n, seed, pbc = np.diag([12.0, 12.5, 30.0]), 50, 23, (True, True, False)
    rng = np.random.default_rng(seed)
    frac = rng.random((n, 3))
    cell = np.asarray(cell, dtype=np.float64)
    return (frac @ cell).astype(np.float32), cell, pbc, np.float32(5.0)


@pytest.mark.parametrize("case", ["orthorhombic_small", "triclinic", "slab"])
def test_neighbors_against_an_all_images_scan(case):
    """The oracle scans |S_a| <= ceil(r_cut / plane spacing) images per periodic axis; an
    independent scan of every image with |S_a| <= 3 (far more than any pair at r < 5 A can use in
    these cells) must find exactly the same (receiver, sender, S) triples and vectors."""
    pos32, cell, pbc, rc = _cell_case(case)
    nb = neighbors(pos32, cell, pbc, rc)
    pos = pos32.astype(np.float64)
    n = len(pos)
    rng3 = [range(-3, 4) if p else range(0, 1) for p in pbc]
    found = {}
    for s0 in rng3[0]:
        for s1 in rng3[1]:
            for s2 in rng3[2]:
                sv = np.array([s0, s1, s2], dtype=np.float64) @ cell
                r = pos[None, :, :] - pos[:, None, :] + sv          # [receiver, sender, 3]
                d = np.sqrt((r * r).sum(-1))
                keep = d < float(rc)
                if (s0, s1, s2) == (0, 0, 0):
                    keep &= ~np.eye(n, dtype=bool)
                for i, j in zip(*np.nonzero(keep)):
                    found[(int(i), int(j), s0, s1, s2)] = r[i, j]
    got = {(int(i), int(j), *map(int, s)): v for i, j, s, v in
           zip(nb["receiver"], nb["sender"], nb["shift"], nb["edge_vec"])}
    assert set(got) == set(found)
    for k, v in got.items():
        assert np.abs(v.astype(np.float64) - found[k]).max() < 1e-5
    # the small cell really has several images of one pair (the case the range rule is for)
    if case == "orthorhombic_small":
        pairs = [(k[0], k[1]) for k in got]
        assert len(pairs) > len(set(pairs))
