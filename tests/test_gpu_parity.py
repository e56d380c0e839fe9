"""GPU parity: every kernel of libetp against the float64 oracle, through the C ABI.

Integer graph arrays must match bit for bit; floating outputs within the per-irrep-block bound
max|gpu - ref| <= 1e-5 max|ref| (grad_edge_vec and forces: over the whole array). Full outputs
on the small workloads (several 32-edge tiles with a ragged tail); sampled receivers/senders,
computed one by one by the oracle, on the full-size ones, in the launch configuration the
benchmark uses.
"""
import os

import numpy as np
import pytest

import workloads
from oracle.conv import conv_forward, conv_vjp
from oracle.graph import forces_from_edge_grads
from oracle.radial import radial
from oracle.conv import ConvSpec
from tests._oracle_side import (assert_blocks_close, assert_close_rel, assert_irrep_blocks_close, forward_ref,
                                full_graph, given_graph, rows_subgraph, sampled_rows, sender_edges, spec_of)

torch = pytest.importorskip("torch")
etp = pytest.importorskip("equivariant_mlip_tensor_edge_b200")

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
N_SAMPLE = 48


@pytest.fixture(scope="module")
def wls():
    cache = {}

    def get(name):
        if name not in cache:
            cache[name] = workloads.make(name)
        return cache[name]
    return get


def _gpu_graph(wl):
    if wl.given_receiver is not None:
        return etp.build_csr(wl.n_nodes, torch.from_numpy(wl.given_receiver).to(DEV),
                             torch.from_numpy(wl.given_sender).to(DEV), torch.from_numpy(wl.given_edge_vec).to(DEV))
    return etp.neighbors(torch.from_numpy(wl.pos).to(DEV), float(wl.r_cut), cell=wl.cell, pbc=wl.pbc)


def _np(t):
    return t.detach().cpu().numpy()


def _conv(wl):
    return etp.EdgeConv(wl.irreps, wl.lmax, wl.irreps, wl.n_basis, float(wl.r_cut))


def _edge_keys(receiver, sender, shift, n_nodes):
    s = np.asarray(shift, np.int64) + 2
    return ((np.asarray(receiver, np.int64) * n_nodes + np.asarray(sender, np.int64)) * 125
            + s[:, 0] * 25 + s[:, 1] * 5 + s[:, 2])


def _gpu_receivers(g):
    return np.repeat(np.arange(g.n_nodes), np.diff(_np(g.row_ptr)))


# ------------------------------------------------------------------ graph

@pytest.mark.parametrize("search", ["default", "bins", "all-pairs"])
@pytest.mark.parametrize("name", ["tiny", "diamond1k"])
def test_neighbors_bit_exact_full(wls, name, search, monkeypatch):
    monkeypatch.setenv("ETP_NEIGHBORS", search)
    wl = wls(name)
    ref = full_graph(wl)
    g = _gpu_graph(wl)
    assert g.n_edges == len(ref["sender"])
    assert np.array_equal(_np(g.row_ptr), ref["row_ptr"])
    assert np.array_equal(_np(g.sender), ref["sender"])
    assert np.array_equal(_np(g.shift), ref["shift"])
    assert np.array_equal(_np(g.edge_vec).view(np.uint32), ref["edge_vec"].view(np.uint32))
    assert np.array_equal(_np(g.t_row_ptr), ref["t_row_ptr"])
    assert np.array_equal(_np(g.t_perm), ref["t_perm"])


class _Cell:
    """A small periodic system for the neighbour paths that the workloads do not reach."""

    def __init__(self, cell, n, seed, r_cut=5.0):
        rng = np.random.default_rng(seed)
        frac = rng.random((n, 3))
        self.cell = np.asarray(cell, dtype=np.float64)
        self.pos = (frac @ self.cell).astype(np.float32)
        self.pbc = (True, True, True)
        self.r_cut = np.float32(r_cut)
        self.n_nodes = n


@pytest.mark.parametrize("search", ["bins", "all-pairs"])
@pytest.mark.parametrize("case", ["orthorhombic_small", "triclinic", "slab"])
def test_neighbors_bit_exact_image_scan(case, search, monkeypatch):
    """Cells where the nearest-image shortcut does not apply: a periodic length below 2 r_cut
    (several images of one pair), a sheared cell, and a slab periodic in two axes only; both the
    binned and the all-pairs search against the oracle."""
    monkeypatch.setenv("ETP_NEIGHBORS", search)
    if case == "orthorhombic_small":
        sysm = _Cell(np.diag([7.1, 7.6, 8.3]), 40, seed=21)
    elif case == "triclinic":
        sysm = _Cell([[11.0, 0.0, 0.0], [3.1, 10.5, 0.0], [-1.7, 2.2, 12.0]], 60, seed=22)
    else:
        sysm = _Cell(np.diag([12.0, 12.5, 30.0]), 50, seed=23)
        sysm.pbc = (True, True, False)
    ref = full_graph(sysm)
    g = etp.neighbors(torch.from_numpy(sysm.pos).to(DEV), float(sysm.r_cut), cell=sysm.cell, pbc=sysm.pbc)
    assert g.n_edges == len(ref["sender"])
    assert np.array_equal(_np(g.row_ptr), ref["row_ptr"])
    assert np.array_equal(_np(g.sender), ref["sender"])
    assert np.array_equal(_np(g.shift), ref["shift"])
    assert np.array_equal(_np(g.edge_vec).view(np.uint32), ref["edge_vec"].view(np.uint32))
    assert np.array_equal(_np(g.t_row_ptr), ref["t_row_ptr"])
    assert np.array_equal(_np(g.t_perm), ref["t_perm"])


def _graph_arrays(g):
    return [_np(a) for a in (g.row_ptr, g.sender, g.shift, g.edge_vec.view(torch.int32), g.t_row_ptr, g.t_perm)]


def _uniform_positions(n, seed, box):
    return (np.random.default_rng(seed).random((n, 3)) * np.asarray(box)).astype(np.float32)


@pytest.mark.parametrize("case", ["diamond8k", "melt32k", "cluster", "slab"])
def test_neighbors_binned_equals_all_pairs(wls, case, monkeypatch):
    """Large systems where the default search bins the atoms: every output of the binned search is
    bit for bit the all-pairs search's (which the oracle pins on the small cells above)."""
    if case in ("diamond8k", "melt32k"):
        wl = wls(case)
        pos, rc, cell, pbc = wl.pos, float(wl.r_cut), wl.cell, wl.pbc
    elif case == "cluster":   # no cell at all
        pos, rc, cell, pbc = _uniform_positions(3000, 31, 40.0), 5.0, None, (False, False, False)
    else:                     # periodic in x and y only, 4000 atoms in a 36 x 36 x 40 slab
        pos, rc, cell, pbc = _uniform_positions(4000, 32, (36.0, 36.0, 40.0)), 5.0, np.diag([36.0, 36.0, 60.0]), \
            (True, True, False)
    pd = torch.from_numpy(np.asarray(pos, np.float32)).to(DEV)
    res = {}
    for search in ("default", "bins", "all-pairs"):
        monkeypatch.setenv("ETP_NEIGHBORS", search)
        res[search] = _graph_arrays(etp.neighbors(pd, rc, cell=cell, pbc=pbc))
    for search in ("default", "bins"):
        for a, b, what in zip(res[search], res["all-pairs"], ("row_ptr", "sender", "shift", "edge_vec", "t_row_ptr", "t_perm")):
            assert np.array_equal(a, b), f"{case}: {search} search differs from all-pairs in {what}"


@pytest.mark.parametrize("name", ["diamond8k", "melt32k"])
def test_neighbors_bit_exact_sampled(wls, name):
    wl = wls(name)
    g = _gpu_graph(wl)
    rng = np.random.default_rng(7)
    sample = np.sort(rng.choice(wl.n_nodes, size=N_SAMPLE, replace=False))
    rows = sampled_rows(wl, sample)
    rp = _np(g.row_ptr)
    snd, shf, vec = _np(g.sender), _np(g.shift), _np(g.edge_vec)
    for i in sample:
        m = rows["receiver"] == i
        a, b = rp[i], rp[i + 1]
        assert b - a == m.sum()
        assert np.array_equal(snd[a:b], rows["sender"][m])
        assert np.array_equal(shf[a:b], rows["shift"][m])
        assert np.array_equal(vec[a:b].view(np.uint32), rows["edge_vec"][m].view(np.uint32))
    # transposed order: edges sent by j = mirror of row j (symmetric test), so counts agree
    trp = _np(g.t_row_ptr)
    for i in sample:
        assert trp[i + 1] - trp[i] == rp[i + 1] - rp[i]
    # t_perm: the stable sort of the canonical edge ids by sender
    tp = _np(g.t_perm)
    s_sorted = snd[tp]
    assert np.all(np.diff(s_sorted) >= 0)
    same = np.diff(s_sorted) == 0
    assert np.all(np.diff(tp)[same] > 0)
    assert np.array_equal(np.sort(tp), np.arange(g.n_edges))


@pytest.mark.parametrize("name", ["sweep1", "sweep2", "sweep3"])
def test_build_csr_bit_exact(wls, name):
    wl = wls(name)
    ref = given_graph(wl)
    g = _gpu_graph(wl)
    assert np.array_equal(_np(g.perm), ref["perm"])
    assert np.array_equal(_np(g.row_ptr), ref["row_ptr"])
    assert np.array_equal(_np(g.sender), ref["sender"])
    assert np.array_equal(_np(g.edge_vec).view(np.uint32), ref["edge_vec"].view(np.uint32))
    assert np.array_equal(_np(g.t_row_ptr), ref["t_row_ptr"])
    assert np.array_equal(_np(g.t_perm), ref["t_perm"])


# ------------------------------------------------------------------ forward

def _inputs(wl, conv):
    x = wl.features()
    W = wl.weights(conv.n_paths)
    return x, W


@pytest.mark.parametrize("name", ["tiny", "diamond1k"])
def test_forward_parity_full(wls, name):
    wl = wls(name)
    conv = _conv(wl)
    spec = spec_of(wl)
    x, W = _inputs(wl, conv)
    g = _gpu_graph(wl)
    out = conv.forward(g, torch.from_numpy(x).to(DEV), torch.from_numpy(W).to(DEV))
    ref = forward_ref(wl, spec, x, W, graph=full_graph(wl))
    assert_blocks_close(_np(out), ref, wl.channels, wl.lmax, f"{name} forward")


@pytest.mark.parametrize("name", ["sweep1", "sweep2", "sweep3", "diamond8k", "melt32k"])
def test_forward_parity_sampled(wls, name):
    wl = wls(name)
    conv = _conv(wl)
    spec = spec_of(wl)
    x, W = _inputs(wl, conv)
    g = _gpu_graph(wl)
    out = _np(conv.forward(g, torch.from_numpy(x).to(DEV), torch.from_numpy(W).to(DEV)))
    rng = np.random.default_rng(11)
    sample = np.sort(rng.choice(wl.n_nodes, size=N_SAMPLE, replace=False))
    if wl.given_receiver is not None:
        ref_g = given_graph(wl)
        ref = conv_forward(spec, ref_g["row_ptr"], ref_g["sender"], ref_g["edge_vec"], x, W, receivers=sample)
    else:
        ref, _ = forward_ref(wl, spec, x, W, sample=sample)
    assert_blocks_close(out[sample], ref, wl.channels, wl.lmax, f"{name} forward (sampled)")


def test_forward_bitwise_deterministic(wls):
    wl = wls("diamond1k")
    conv = _conv(wl)
    x, W = _inputs(wl, conv)
    g = _gpu_graph(wl)
    xt, Wt = torch.from_numpy(x).to(DEV), torch.from_numpy(W).to(DEV)
    a = conv.forward(g, xt, Wt).clone()
    b = conv.forward(g, xt, Wt)
    assert torch.equal(a, b)


def test_radial_weights_parity(wls):
    wl = wls("diamond1k")
    conv = _conv(wl)
    _, W = _inputs(wl, conv)
    g = _gpu_graph(wl)
    w = _np(conv.radial_weights(g.edge_vec, torch.from_numpy(W).to(DEV)))
    ref_g = full_graph(wl)
    vec = ref_g["edge_vec"].astype(np.float64)
    rad = radial(np.linalg.norm(vec, axis=1), 8, np.float64(np.float32(wl.r_cut)))
    ref = np.einsum("eb,bpc->epc", rad, W.astype(np.float64))
    assert_close_rel(w, ref, "radial weights")


# ------------------------------------------------------------------ backward

@pytest.mark.parametrize("name", ["tiny", "diamond1k"])
def test_backward_parity_full(wls, name):
    wl = wls(name)
    conv = _conv(wl)
    spec = spec_of(wl)
    x, W = _inputs(wl, conv)
    gout = wl.cotangent()
    g = _gpu_graph(wl)
    gx, gv = conv.backward(g, torch.from_numpy(x).to(DEV), torch.from_numpy(W).to(DEV),
                           torch.from_numpy(gout).to(DEV))
    ref_g = full_graph(wl)
    rgx, rgv = conv_vjp(spec, ref_g["row_ptr"], ref_g["sender"], ref_g["edge_vec"], x, W, gout)
    assert_blocks_close(_np(gx), rgx, wl.channels, wl.lmax, f"{name} grad_x")
    assert_close_rel(_np(gv), rgv, f"{name} grad_edge_vec")
    # forces from the edge gradients
    f = _np(etp.forces(g, gv))
    rf = forces_from_edge_grads(rgv, ref_g["receiver"], ref_g["sender"], wl.n_nodes)
    assert_close_rel(f, rf, f"{name} forces")
    # only one of the two outputs
    gx2, none = conv.backward(g, torch.from_numpy(x).to(DEV), torch.from_numpy(W).to(DEV),
                              torch.from_numpy(gout).to(DEV), want_grad_vec=False)
    assert none is None and torch.equal(gx2, gx)
    none, gv2 = conv.backward(g, torch.from_numpy(x).to(DEV), torch.from_numpy(W).to(DEV),
                              torch.from_numpy(gout).to(DEV), want_grad_x=False)
    assert none is None and torch.equal(gv2, gv)


@pytest.mark.parametrize("name", ["diamond8k", "melt32k"])
def test_backward_parity_sampled(wls, name):
    wl = wls(name)
    conv = _conv(wl)
    spec = spec_of(wl)
    x, W = _inputs(wl, conv)
    gout = wl.cotangent()
    g = _gpu_graph(wl)
    gx, gv = conv.backward(g, torch.from_numpy(x).to(DEV), torch.from_numpy(W).to(DEV),
                           torch.from_numpy(gout).to(DEV))
    gx, gv = _np(gx), _np(gv)
    rng = np.random.default_rng(13)
    sample = np.sort(rng.choice(wl.n_nodes, size=N_SAMPLE // 2, replace=False))
    rows = sampled_rows(wl, sample)
    recv, send, shift, vec = sender_edges(rows)
    rp, snd, v = rows_subgraph(wl.n_nodes, recv, send, vec)
    rgx, rgv = conv_vjp(spec, rp, snd, v, x, W, gout)
    assert_blocks_close(gx[sample], rgx[sample], wl.channels, wl.lmax, f"{name} grad_x (sampled)")
    keys = _edge_keys(_gpu_receivers(g), _np(g.sender), _np(g.shift), wl.n_nodes)
    want = _edge_keys(recv, send, shift, wl.n_nodes)
    pos = np.searchsorted(keys, want)
    assert np.array_equal(keys[pos], want)
    assert_close_rel(gv[pos], rgv, f"{name} grad_edge_vec (sampled)")


def test_autograd_function_matches_backward(wls):
    wl = wls("tiny")
    conv = _conv(wl)
    x, W = _inputs(wl, conv)
    g = _gpu_graph(wl)
    fn = etp.edge_conv_function()
    xt = torch.from_numpy(x).to(DEV).requires_grad_(True)
    vt = g.edge_vec.clone().requires_grad_(True)
    Wt = torch.from_numpy(W).to(DEV)
    out = fn.apply(conv, g, xt, vt, Wt)
    gout = torch.from_numpy(wl.cotangent()).to(DEV)
    (out * gout).sum().backward()
    gx, gv = conv.backward(g, xt.detach(), Wt, gout)
    assert torch.equal(xt.grad, gx) and torch.equal(vt.grad, gv)


# ------------------------------------------------------------------ edge cases

def test_empty_graph_and_isolated_nodes():
    conv = etp.EdgeConv("8x0e+8x1o", 1, "8x0e+8x1o", 8, 4.0)
    pos = torch.tensor([[0.0, 0.0, 0.0], [10.0, 0.0, 0.0], [20.0, 0.0, 0.0]], device=DEV)
    g = etp.neighbors(pos, 4.0)
    assert g.n_edges == 0
    x = torch.randn(3, 32, device=DEV)
    W = torch.randn(8, conv.n_paths, 8, device=DEV)
    out = conv.forward(g, x, W, out=torch.full((3, 32), 7.0, device=DEV))
    assert torch.count_nonzero(out) == 0
    gx, gv = conv.backward(g, x, W, torch.randn(3, 32, device=DEV),
                           grad_x=torch.full((3, 32), 7.0, device=DEV))
    assert torch.count_nonzero(gx) == 0 and gv.numel() == 0
    f = etp.forces(g, gv)
    assert torch.count_nonzero(f) == 0
    # one node, no edges
    g1 = etp.neighbors(pos[:1], 4.0)
    assert g1.n_edges == 0 and torch.count_nonzero(conv.forward(g1, x[:1], W)) == 0


def test_edges_beyond_cutoff_contribute_zero():
    conv = etp.EdgeConv("4x0e+4x1o", 1, "4x0e+4x1o", 8, 3.0)
    recv = torch.tensor([0, 0, 1], device=DEV)
    send = torch.tensor([1, 1, 0], device=DEV)
    vec = torch.tensor([[3.0, 0.0, 0.0], [0.0, 4.0, 0.0], [0.0, 0.0, -3.5]], device=DEV)
    g = etp.build_csr(2, recv, send, vec)
    out = conv.forward(g, torch.randn(2, 16, device=DEV), torch.randn(8, conv.n_paths, 4, device=DEV))
    assert torch.count_nonzero(out) == 0


def test_validation_rejects_corrupt_graph(wls, monkeypatch):
    wl = wls("tiny")
    conv = _conv(wl)
    x, W = _inputs(wl, conv)
    g = _gpu_graph(wl)
    bad_ptr = g.row_ptr.clone()
    bad_ptr[5] = bad_ptr[6] + 3          # not monotone
    bad = etp.Graph(g.n_nodes, g.n_edges, bad_ptr, g.sender, g.edge_vec, g.t_row_ptr, g.t_perm)
    monkeypatch.setenv("ETP_VALIDATE", "1")
    out = torch.full((wl.n_nodes, wl.dim), 3.0, device=DEV)
    with pytest.raises(etp.EtpError) as ei:
        conv.forward(bad, torch.from_numpy(x).to(DEV), torch.from_numpy(W).to(DEV), out=out)
    assert ei.value.status == 4
    assert bool((out == 3.0).all())
    bad_sender = g.sender.clone()
    bad_sender[0] = wl.n_nodes + 5
    bad2 = etp.Graph(g.n_nodes, g.n_edges, g.row_ptr, bad_sender, g.edge_vec, g.t_row_ptr, g.t_perm)
    with pytest.raises(etp.EtpError):
        conv.backward(bad2, torch.from_numpy(x).to(DEV), torch.from_numpy(W).to(DEV),
                      torch.from_numpy(wl.cotangent()).to(DEV))
    bad_tp = g.t_perm.clone()
    bad_tp[0] = bad_tp[1]
    bad3 = etp.Graph(g.n_nodes, g.n_edges, g.row_ptr, g.sender, g.edge_vec, g.t_row_ptr, bad_tp)
    with pytest.raises(etp.EtpError):
        conv.backward(bad3, torch.from_numpy(x).to(DEV), torch.from_numpy(W).to(DEV),
                      torch.from_numpy(wl.cotangent()).to(DEV))
    monkeypatch.delenv("ETP_VALIDATE")
    conv.forward(g, torch.from_numpy(x).to(DEV), torch.from_numpy(W).to(DEV), out=out)
    torch.cuda.synchronize()


def test_build_csr_rejects_out_of_range():
    recv = torch.tensor([0, 3], device=DEV)
    send = torch.tensor([1, 0], device=DEV)
    vec = torch.zeros(2, 3, device=DEV)
    with pytest.raises(etp.EtpError) as ei:
        etp.build_csr(2, recv, send, vec)
    assert ei.value.status == 4


def test_no_cpu_fallback():
    conv = etp.EdgeConv("8x0e+8x1o", 1, "8x0e+8x1o", 8, 4.0)
    with pytest.raises(ValueError):
        conv.radial_weights(torch.zeros(3, 3), torch.zeros(8, conv.n_paths, 8))
    assert os.path.exists(etp.LIB_PATH)


# ------------------------------------------------------------------ forward kernels: both implementations

@pytest.mark.parametrize("impl", ["default", "edge", "generic"])
@pytest.mark.parametrize("name", ["tiny", "diamond1k"])
def test_forward_both_kernels(wls, name, impl, monkeypatch):
    if impl != "default":
        monkeypatch.setenv("ETP_FORWARD", impl)
    monkeypatch.setenv("ETP_VALIDATE", "1")      # graph checks + device pipeline status word
    wl = wls(name)
    conv = _conv(wl)
    x, W = _inputs(wl, conv)
    g = _gpu_graph(wl)
    out = conv.forward(g, torch.from_numpy(x).to(DEV), torch.from_numpy(W).to(DEV))
    ref = forward_ref(wl, spec_of(wl), x, W, graph=full_graph(wl))
    assert_blocks_close(_np(out), ref, wl.channels, wl.lmax, f"{name} forward ({impl})")


def _random_graph(n_nodes, degrees, seed, r_max=4.5):
    rng = np.random.default_rng(seed)
    recv = np.repeat(np.arange(n_nodes), degrees)
    send = rng.integers(0, n_nodes, size=len(recv))
    d = rng.standard_normal((len(recv), 3))
    d /= np.linalg.norm(d, axis=1, keepdims=True)
    vec = (d * rng.uniform(0.5, r_max, size=(len(recv), 1))).astype(np.float32)
    return recv, send, vec


@pytest.mark.parametrize("lmax,c", [(1, 20), (2, 24), (3, 8)])
def test_forward_ragged_degrees_and_channels(lmax, c):
    """Degrees 0..300 (several 128-edge rounds, empty rows, ragged tiles) and C not a multiple of 16."""
    from oracle.conv import ConvSpec
    irr = "+".join(f"{c}x{l}{'eo'[l % 2]}" for l in range(lmax + 1))
    n = 13
    degrees = np.array([0, 1, 31, 32, 33, 127, 128, 129, 300, 5, 0, 64, 97])
    recv, send, vec = _random_graph(n, degrees, seed=lmax)
    conv = etp.EdgeConv(irr, lmax, irr, 8, 5.0)
    spec = ConvSpec(irr, lmax, irr, 8, 5.0)
    rng = np.random.default_rng(100 + lmax)
    x = rng.standard_normal((n, spec.dim_in)).astype(np.float32)
    W = (rng.standard_normal((8, len(spec.paths), c)) / np.sqrt(8)).astype(np.float32)
    g = etp.build_csr(n, torch.from_numpy(recv).to(DEV), torch.from_numpy(send).to(DEV),
                      torch.from_numpy(vec).to(DEV))
    out = _np(conv.forward(g, torch.from_numpy(x).to(DEV), torch.from_numpy(W).to(DEV)))
    order = np.lexsort((send, recv))
    rp = np.concatenate([[0], np.cumsum(degrees)])
    ref = conv_forward(spec, rp, send[order], vec[order], x, W)
    assert np.all(out[degrees == 0] == 0.0)
    assert_blocks_close(out, ref, c, lmax, f"ragged forward lmax={lmax} C={c}")


# ------------------------------------------------------------------ backward kernels: both implementations

@pytest.mark.parametrize("impl", ["tc", "generic"])
@pytest.mark.parametrize("name", ["tiny", "diamond1k"])
def test_backward_both_kernels(wls, name, impl, monkeypatch):
    if impl == "generic":
        monkeypatch.setenv("ETP_BACKWARD", "generic")
    monkeypatch.setenv("ETP_VALIDATE", "1")      # graph checks + device pipeline status word
    wl = wls(name)
    conv = _conv(wl)
    spec = spec_of(wl)
    x, W = _inputs(wl, conv)
    gout = wl.cotangent()
    g = _gpu_graph(wl)
    args = (g, torch.from_numpy(x).to(DEV), torch.from_numpy(W).to(DEV), torch.from_numpy(gout).to(DEV))
    gx, gv = conv.backward(*args)
    ref_g = full_graph(wl)
    rgx, rgv = conv_vjp(spec, ref_g["row_ptr"], ref_g["sender"], ref_g["edge_vec"], x, W, gout)
    assert_blocks_close(_np(gx), rgx, wl.channels, wl.lmax, f"{name} grad_x ({impl})")
    assert_close_rel(_np(gv), rgv, f"{name} grad_edge_vec ({impl})")
    gx2, gv2 = conv.backward(*args)
    assert torch.equal(gx, gx2) and torch.equal(gv, gv2), "backward is not bitwise deterministic"


def _skewed_graph(n_nodes, degrees, seed, hub, silent, r_max=4.5):
    """Receiver degrees as given; about half of all edges sent by `hub`, none by `silent`."""
    rng = np.random.default_rng(seed)
    recv = np.repeat(np.arange(n_nodes), degrees)
    others = np.array([i for i in range(n_nodes) if i != silent])
    send = np.where(rng.random(len(recv)) < 0.5, hub, rng.choice(others, size=len(recv)))
    d = rng.standard_normal((len(recv), 3))
    d /= np.linalg.norm(d, axis=1, keepdims=True)
    vec = (d * rng.uniform(0.5, r_max, size=(len(recv), 1))).astype(np.float32)
    return recv, send, vec


@pytest.mark.parametrize("lmax,c", [(1, 20), (2, 24), (3, 8), (3, 36)])
def test_backward_ragged_degrees_and_channels(lmax, c):
    """Sender degrees from 0 to several 128-edge rounds, ragged tiles, C not a multiple of 16."""
    from oracle.conv import ConvSpec
    irr = "+".join(f"{c}x{l}{'eo'[l % 2]}" for l in range(lmax + 1))
    n = 13
    degrees = np.array([0, 1, 31, 32, 33, 127, 128, 129, 300, 5, 0, 64, 97])
    recv, send, vec = _skewed_graph(n, degrees, seed=10 + lmax, hub=3, silent=10)
    conv = etp.EdgeConv(irr, lmax, irr, 8, 5.0)
    spec = ConvSpec(irr, lmax, irr, 8, 5.0)
    rng = np.random.default_rng(200 + lmax)
    x = rng.standard_normal((n, spec.dim_in)).astype(np.float32)
    W = (rng.standard_normal((8, len(spec.paths), c)) / np.sqrt(8)).astype(np.float32)
    gout = rng.standard_normal((n, spec.dim_out)).astype(np.float32)
    g = etp.build_csr(n, torch.from_numpy(recv).to(DEV), torch.from_numpy(send).to(DEV),
                      torch.from_numpy(vec).to(DEV))
    gx, gv = conv.backward(g, torch.from_numpy(x).to(DEV), torch.from_numpy(W).to(DEV),
                           torch.from_numpy(gout).to(DEV))
    gx, gv = _np(gx), _np(gv)
    order = np.lexsort((send, recv))
    rp = np.concatenate([[0], np.cumsum(degrees)])
    rgx, rgv = conv_vjp(spec, rp, send[order], vec[order], x, W, gout)
    assert np.all(gx[10] == 0.0)
    assert_blocks_close(gx, rgx, c, lmax, f"ragged grad_x lmax={lmax} C={c}")
    assert_close_rel(gv, rgv, f"ragged grad_edge_vec lmax={lmax} C={c}")


# ------------------------------------------------------------------ weight gradient dL/dW

def _weight_grad_ref(wl, spec, x, gout):
    from oracle.conv import conv_vjp_weights
    ref_g = full_graph(wl)
    return conv_vjp_weights(spec, ref_g["row_ptr"], ref_g["sender"], ref_g["edge_vec"], x, gout)


@pytest.mark.parametrize("name", ["tiny", "diamond1k"])
def test_weight_grad_parity_full(wls, name):
    wl = wls(name)
    conv = _conv(wl)
    spec = spec_of(wl)
    x, W = _inputs(wl, conv)
    gout = wl.cotangent()
    g = _gpu_graph(wl)
    xd, gd = torch.from_numpy(x).to(DEV), torch.from_numpy(gout).to(DEV)
    dw = conv.backward_weights(g, xd, gd)
    ref = _weight_grad_ref(wl, spec, x, gout)
    assert_close_rel(_np(dw), ref, f"{name} dL/dW")
    assert torch.equal(dw, conv.backward_weights(g, xd, gd)), "weight gradient is not bitwise deterministic"


@pytest.mark.parametrize("name", ["diamond8k", "melt32k"])
def test_weight_grad_adjoint_at_full_size(wls, name):
    """At sizes the oracle cannot finish: the forward is linear in W, so <dL/dW, V> = <g, F(W = V)>
    for a random V, with both sides from the GPU (the forward is checked against the oracle)."""
    wl = wls(name)
    conv = _conv(wl)
    x, _ = _inputs(wl, conv)
    g = _gpu_graph(wl)
    xd = torch.from_numpy(x).to(DEV)
    gd = torch.from_numpy(wl.cotangent()).to(DEV)
    dw = conv.backward_weights(g, xd, gd).double()
    rng = np.random.default_rng(17)
    v = torch.from_numpy(rng.standard_normal(tuple(dw.shape)).astype(np.float32)).to(DEV)
    out = conv.forward(g, xd, v).double()
    lhs = float((dw * v.double()).sum())
    rhs = float((gd.double() * out).sum())
    scale = float((dw.abs() * v.double().abs()).sum())
    assert abs(lhs - rhs) <= 1e-5 * scale, (lhs, rhs, scale)


@pytest.mark.parametrize("lmax,c", [(1, 20), (2, 24), (3, 8), (3, 36)])
def test_weight_grad_ragged_degrees_and_channels(lmax, c):
    from oracle.conv import ConvSpec, conv_vjp_weights
    irr = "+".join(f"{c}x{l}{'eo'[l % 2]}" for l in range(lmax + 1))
    n = 13
    degrees = np.array([0, 1, 31, 32, 33, 127, 128, 129, 300, 5, 0, 64, 97])
    recv, send, vec = _skewed_graph(n, degrees, seed=20 + lmax, hub=3, silent=10)
    conv = etp.EdgeConv(irr, lmax, irr, 8, 5.0)
    spec = ConvSpec(irr, lmax, irr, 8, 5.0)
    rng = np.random.default_rng(300 + lmax)
    x = rng.standard_normal((n, spec.dim_in)).astype(np.float32)
    gout = rng.standard_normal((n, spec.dim_out)).astype(np.float32)
    g = etp.build_csr(n, torch.from_numpy(recv).to(DEV), torch.from_numpy(send).to(DEV),
                      torch.from_numpy(vec).to(DEV))
    dw = _np(conv.backward_weights(g, torch.from_numpy(x).to(DEV), torch.from_numpy(gout).to(DEV)))
    order = np.lexsort((send, recv))
    rp = np.concatenate([[0], np.cumsum(degrees)])
    ref = conv_vjp_weights(spec, rp, send[order], vec[order], x, gout)
    assert_close_rel(dw, ref, f"ragged dL/dW lmax={lmax} C={c}")


def test_weight_grad_empty_graph_and_autograd(wls):
    wl = wls("tiny")
    conv = _conv(wl)
    x, W = _inputs(wl, conv)
    # no edges: the gradient is zero
    n = 5
    empty = etp.build_csr(n, torch.zeros(0, dtype=torch.int32, device=DEV), torch.zeros(0, dtype=torch.int32, device=DEV),
                          torch.zeros((0, 3), dtype=torch.float32, device=DEV))
    xe = torch.randn(n, conv.info["dim_in"], device=DEV)
    ge = torch.randn(n, conv.info["dim_out"], device=DEV)
    dw0 = conv.backward_weights(empty, xe, ge)
    assert torch.count_nonzero(dw0) == 0
    # autograd: W.grad equals backward_weights
    g = _gpu_graph(wl)
    fn = etp.edge_conv_function()
    xt = torch.from_numpy(x).to(DEV)
    Wt = torch.from_numpy(W).to(DEV).requires_grad_(True)
    out = fn.apply(conv, g, xt, g.edge_vec, Wt)
    gout = torch.from_numpy(wl.cotangent()).to(DEV)
    (out * gout).sum().backward()
    assert torch.equal(Wt.grad, conv.backward_weights(g, xt, gout))


# ------------------------------------------------------------------ path-subset forward

@pytest.mark.parametrize("lmax,c", [(1, 8), (1, 32), (1, 64), (2, 8), (2, 20), (2, 36), (2, 64)])
def test_forward_path_subset_kernel_ragged(lmax, c, monkeypatch):
    """The default forward for l_max <= 2 and C <= 64 (channel-major, two path subsets): empty rows
    at both ends and in between, receivers whose edges span several CTAs (the kernel cuts the edge
    list into equal ranges of at least 64 edges, so the 127..300-edge rows cross range
    boundaries), channel counts that leave lanes idle (8, 20, 36); compared with the oracle and
    bitwise reproducible."""
    from oracle.conv import ConvSpec
    monkeypatch.setenv("ETP_VALIDATE", "1")
    irr = "+".join(f"{c}x{l}{'eo'[l % 2]}" for l in range(lmax + 1))
    degrees = np.array([0, 0, 1, 31, 32, 33, 0, 127, 128, 129, 300, 5, 0, 64, 97, 15, 17, 0])
    n = len(degrees)
    recv, send, vec = _random_graph(n, degrees, seed=70 + lmax + c)
    conv = etp.EdgeConv(irr, lmax, irr, 8, 5.0)
    spec = ConvSpec(irr, lmax, irr, 8, 5.0)
    rng = np.random.default_rng(700 + lmax + c)
    x = rng.standard_normal((n, spec.dim_in)).astype(np.float32)
    W = (rng.standard_normal((8, len(spec.paths), c)) / np.sqrt(8)).astype(np.float32)
    g = etp.build_csr(n, torch.from_numpy(recv).to(DEV), torch.from_numpy(send).to(DEV),
                      torch.from_numpy(vec).to(DEV))
    xd, Wd = torch.from_numpy(x).to(DEV), torch.from_numpy(W).to(DEV)
    out = conv.forward(g, xd, Wd)
    again = conv.forward(g, xd, Wd)
    assert torch.equal(out, again), "path-subset forward is not bitwise deterministic"
    order = np.lexsort((send, recv))
    rp = np.concatenate([[0], np.cumsum(degrees)])
    ref = conv_forward(spec, rp, send[order], vec[order], x, W)
    o = _np(out)
    assert np.all(o[degrees == 0] == 0.0)
    assert_blocks_close(o, ref, c, lmax, f"path-subset forward lmax={lmax} C={c}")


# ------------------------------------------------------------------ per-edge path masks

@pytest.mark.parametrize("name", ["tiny", "diamond1k"])
def test_path_mask_forward_backward_parity(wls, name, monkeypatch):
    monkeypatch.setenv("ETP_VALIDATE", "1")
    wl = wls(name)
    conv = _conv(wl)
    spec = spec_of(wl)
    x, W = _inputs(wl, conv)
    gout = wl.cotangent()
    g = _gpu_graph(wl)
    ref_g = full_graph(wl)
    n_p = conv.n_paths
    rng = np.random.default_rng(31)
    mask = rng.integers(0, 1 << n_p, size=g.n_edges).astype(np.int64)
    mask[: g.n_edges // 3] = (1 << n_p) - 1          # some edges keep every path
    md = torch.from_numpy(mask.astype(np.int32)).to(DEV)
    xd, Wd, gd = torch.from_numpy(x).to(DEV), torch.from_numpy(W).to(DEV), torch.from_numpy(gout).to(DEV)
    out = conv.forward(g, xd, Wd, path_mask=md)
    ref = conv_forward(spec, ref_g["row_ptr"], ref_g["sender"], ref_g["edge_vec"], x, W, path_mask=mask)
    assert_blocks_close(_np(out), ref, wl.channels, wl.lmax, f"{name} masked forward")
    gx, gv = conv.backward(g, xd, Wd, gd, path_mask=md)
    rgx, rgv = conv_vjp(spec, ref_g["row_ptr"], ref_g["sender"], ref_g["edge_vec"], x, W, gout, path_mask=mask)
    assert_blocks_close(_np(gx), rgx, wl.channels, wl.lmax, f"{name} masked grad_x")
    assert_close_rel(_np(gv), rgv, f"{name} masked grad_edge_vec")


def test_path_mask_all_ones_and_zero(wls, monkeypatch):
    """All bits set is the unmasked call of the same (edge-major) kernels, bit for bit; no bits set
    gives zeros. Masked calls run the edge-major kernels, so the unmasked forward is pinned to it."""
    monkeypatch.setenv("ETP_FORWARD", "edge")
    wl = wls("diamond1k")
    conv = _conv(wl)
    x, W = _inputs(wl, conv)
    g = _gpu_graph(wl)
    xd, Wd = torch.from_numpy(x).to(DEV), torch.from_numpy(W).to(DEV)
    gd = torch.from_numpy(wl.cotangent()).to(DEV)
    ones = torch.full((g.n_edges,), (1 << conv.n_paths) - 1, dtype=torch.int32, device=DEV)
    zero = torch.zeros(g.n_edges, dtype=torch.int32, device=DEV)
    assert torch.equal(conv.forward(g, xd, Wd, path_mask=ones), conv.forward(g, xd, Wd))
    assert torch.count_nonzero(conv.forward(g, xd, Wd, path_mask=zero)) == 0
    gx1, gv1 = conv.backward(g, xd, Wd, gd, path_mask=ones)
    gx0, gv0 = conv.backward(g, xd, Wd, gd)
    assert torch.equal(gx1, gx0) and torch.equal(gv1, gv0)
    gxz, gvz = conv.backward(g, xd, Wd, gd, path_mask=zero)
    assert torch.count_nonzero(gxz) == 0 and torch.count_nonzero(gvz) == 0


# ------------------------------------------------------------------ node-local product ladder

@pytest.mark.parametrize("lmax,c,n,nu", [(1, 128, 4096, 3), (2, 128, 4096, 3), (3, 128, 4096, 2), (2, 64, 37, 5),
                                        (3, 8, 37, 4), (1, 4, 5, 1)])
def test_node_ladder_parity(lmax, c, n, nu):
    """The node-local product ladder against the oracle: the pages' 4096-node x 128-channel case and
    small ragged ones, correlation orders 1..5."""
    from oracle.product import node_ladder, product_paths
    rng = np.random.default_rng(600 + 10 * lmax + nu)
    dim = (lmax + 1) ** 2 * c
    n_p = len(product_paths(lmax))
    A = rng.standard_normal((n, dim)).astype(np.float32)
    Ws = (rng.standard_normal((nu - 1, n_p, c)) / np.sqrt(n_p)).astype(np.float32)
    out = etp.node_ladder(torch.from_numpy(A).to(DEV), torch.from_numpy(Ws).to(DEV), lmax)
    ref = node_ladder(lmax, c, A, Ws)
    assert_blocks_close(_np(out), ref, c, lmax, f"node ladder lmax={lmax} C={c} nu={nu}")


# ------------------------------------------------------------------ general irreps

GENERAL = [
    ("128x0e+64x1o+32x2e+32x3o", 3, "128x0e+64x1o+32x2e+32x3o"),        # NequIP-L channel counts
    ("4x0e+3x1o+3x1e+4x2e+2x2o+3x3o+4x4e", 4, "4x0e+3x1o+3x1e+4x2e+2x2o+3x3o+4x4e"),
    ("16x0e+16x1o+16x1e+16x2e+16x2o", 2, "16x0e+16x1o+16x1e+16x2e+16x2o"),   # odd l1 + l2 + l3 paths
    ("32x0e+32x1o+32x2e+32x3o+32x4e", 4, "32x0e+32x1o+32x2e+32x3o+32x4e"),   # rank 4
    ("16x0e+16x1o", 2, "16x0e+16x1o+16x1e+16x2e"),                         # irreps_out != irreps_in
    ("6x0e+6x1o+6x2e", 2, "6x0e+6x1o+6x2e"),                               # C not a multiple of 4
    ("8x0e+4x2e", 0, "8x0e+4x1o"),         # an input block no path reads, an output block none writes
]


def _general_inputs(spec, n, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, spec.dim_in)).astype(np.float32)
    W = (rng.standard_normal((8, spec.weight_numel)) / np.sqrt(len(spec.paths))).astype(np.float32)
    gout = rng.standard_normal((n, spec.dim_out)).astype(np.float32)
    return x, W, gout


@pytest.mark.parametrize("irin,sh,irout", GENERAL)
def test_general_irreps_parity_full(wls, irin, sh, irout):
    """Forward and backward of general irreps handles against the oracle on the whole small cell."""
    wl = wls("tiny")
    conv = etp.EdgeConv(irin, sh, irout, 8, float(wl.r_cut))
    assert conv.info["general"] == 1
    spec = ConvSpec(irin, sh, irout, 8, float(wl.r_cut))
    x, W, gout = _general_inputs(spec, wl.n_nodes, len(irin) + sh)
    g = _gpu_graph(wl)
    ref_g = full_graph(wl)
    xd, Wd, gd = (torch.from_numpy(a).to(DEV) for a in (x, W, gout))
    out = conv.forward(g, xd, Wd)
    ref = conv_forward(spec, ref_g["row_ptr"], ref_g["sender"], ref_g["edge_vec"], x, W)
    assert_irrep_blocks_close(_np(out), ref, spec, "out", f"{irin} forward")
    gx, gv = conv.backward(g, xd, Wd, gd)
    rgx, rgv = conv_vjp(spec, ref_g["row_ptr"], ref_g["sender"], ref_g["edge_vec"], x, W, gout)
    assert_irrep_blocks_close(_np(gx), rgx, spec, "in", f"{irin} grad_x")
    assert_close_rel(_np(gv), rgv, f"{irin} grad_edge_vec")
    # the no-workspace entry point runs the same kernel
    out2 = torch.empty_like(out)
    st = etp.load_library().etp_forward_noalloc(conv._h, g.n_nodes, g.n_edges, etp._ptr(g.row_ptr),
                                                etp._ptr(g.sender), etp._ptr(g.edge_vec), etp._ptr(xd),
                                                etp._ptr(Wd), etp._ptr(out2), etp._stream(xd.device))
    assert st == 0 and torch.equal(out2, out)
    # deterministic
    assert torch.equal(conv.forward(g, xd, Wd), out)


def test_general_irreps_parity_sampled_full_size(wls):
    """NequIP-L channel counts (128x0e+64x1o+32x2e+32x3o, harmonics to l = 3) on the 1000-atom
    diamond cell: sampled receivers (forward) and senders (backward), computed one by one."""
    wl = wls("diamond1k")
    irr = "128x0e+64x1o+32x2e+32x3o"
    conv = etp.EdgeConv(irr, 3, irr, 8, float(wl.r_cut))
    spec = ConvSpec(irr, 3, irr, 8, float(wl.r_cut))
    x, W, gout = _general_inputs(spec, wl.n_nodes, 77)
    g = _gpu_graph(wl)
    xd, Wd, gd = (torch.from_numpy(a).to(DEV) for a in (x, W, gout))
    out = _np(conv.forward(g, xd, Wd))
    rng = np.random.default_rng(17)
    sample = np.sort(rng.choice(wl.n_nodes, size=N_SAMPLE // 2, replace=False))
    ref, _ = forward_ref(wl, spec, x, W, sample=sample)
    assert_irrep_blocks_close(out[sample], ref, spec, "out", "NequIP-L forward (sampled)")
    gx, gv = conv.backward(g, xd, Wd, gd)
    gx, gv = _np(gx), _np(gv)
    rows = sampled_rows(wl, sample)
    recv, send, shift, vec = sender_edges(rows)
    rp, snd, v = rows_subgraph(wl.n_nodes, recv, send, vec)
    rgx, rgv = conv_vjp(spec, rp, snd, v, x, W, gout)
    assert_irrep_blocks_close(gx[sample], rgx[sample], spec, "in", "NequIP-L grad_x (sampled)")
    keys = _edge_keys(_gpu_receivers(g), _np(g.sender), _np(g.shift), wl.n_nodes)
    want = _edge_keys(recv, send, shift, wl.n_nodes)
    pos = np.searchsorted(keys, want)
    assert np.array_equal(keys[pos], want)
    assert_close_rel(gv[pos], rgv, "NequIP-L grad_edge_vec (sampled)")


@pytest.mark.parametrize("impl", ["tc", "fp32"])
@pytest.mark.parametrize("irin,sh,irout", GENERAL)
def test_general_irreps_forward_ragged_both_kernels(irin, sh, irout, impl, monkeypatch):
    """The general forward with its radial projection on the tensor cores (the default) and on the
    FP32 pipe (ETP_GEN_FORWARD=fp32): degrees 0..150 (empty rows, one edge, quads and ragged tails
    of the 32-edge rounds, several rounds) against the oracle, with the status word checked."""
    if impl == "fp32":
        monkeypatch.setenv("ETP_GEN_FORWARD", "fp32")
    monkeypatch.setenv("ETP_VALIDATE", "1")
    n = 12
    degrees = np.array([0, 1, 3, 4, 5, 31, 32, 33, 0, 64, 97, 150])
    recv, send, vec = _random_graph(n, degrees, seed=len(irin) + sh)
    conv = etp.EdgeConv(irin, sh, irout, 8, 5.0)
    spec = ConvSpec(irin, sh, irout, 8, 5.0)
    x, W, _ = _general_inputs(spec, n, 5 + sh)
    g = etp.build_csr(n, torch.from_numpy(recv).to(DEV), torch.from_numpy(send).to(DEV),
                      torch.from_numpy(vec).to(DEV))
    xd, Wd = torch.from_numpy(x).to(DEV), torch.from_numpy(W).to(DEV)
    ws = torch.empty(conv.workspace_bytes(n, g.n_edges), dtype=torch.uint8, device=DEV)
    out = conv.forward(g, xd, Wd, workspace=ws)
    order = np.lexsort((send, recv))
    rp = np.concatenate([[0], np.cumsum(degrees)])
    ref = conv_forward(spec, rp, send[order], vec[order], x, W)
    on = _np(out)
    assert np.all(on[degrees == 0] == 0.0)
    assert_irrep_blocks_close(on, ref, spec, "out", f"{irin} ragged forward ({impl})")
    assert torch.equal(conv.forward(g, xd, Wd, workspace=ws), out)   # bitwise repeatable
    conv.check_status(DEV)


def test_general_irreps_forward_kernels_differ_only_by_rounding(wls, monkeypatch):
    """NequIP-L on the 1000-atom cell: the tensor-core general forward (default) and the FP32 one
    agree to rounding but not bit for bit (so the default really is the tensor-core kernel), and
    the no-workspace entry point runs the default kernel."""
    wl = wls("diamond1k")
    irr = "128x0e+64x1o+32x2e+32x3o"
    conv = etp.EdgeConv(irr, 3, irr, 8, float(wl.r_cut))
    spec = ConvSpec(irr, 3, irr, 8, float(wl.r_cut))
    x, W, _ = _general_inputs(spec, wl.n_nodes, 78)
    g = _gpu_graph(wl)
    xd, Wd = torch.from_numpy(x).to(DEV), torch.from_numpy(W).to(DEV)
    out_tc = conv.forward(g, xd, Wd)
    out_nw = torch.empty_like(out_tc)
    st = etp.load_library().etp_forward_noalloc(conv._h, g.n_nodes, g.n_edges, etp._ptr(g.row_ptr),
                                                etp._ptr(g.sender), etp._ptr(g.edge_vec), etp._ptr(xd),
                                                etp._ptr(Wd), etp._ptr(out_nw), etp._stream(xd.device))
    assert st == 0 and torch.equal(out_nw, out_tc)
    monkeypatch.setenv("ETP_GEN_FORWARD", "fp32")
    out_fp = conv.forward(g, xd, Wd)
    assert not torch.equal(out_fp, out_tc)
    # each is within 1e-5 max|ref| of the oracle (the tests above), so within twice that of the other
    assert_irrep_blocks_close(_np(out_tc), _np(out_fp).astype(np.float64), spec, "out",
                              "NequIP-L tensor-core vs FP32 forward", tol=2e-5)


@pytest.mark.parametrize("irr,sh", [("64x0e+64x1o+64x1e+64x2e+64x2o", 2), ("32x0e+32x1o+32x2e+32x3o+32x4e", 4)])
def test_general_irreps_forward_tc_full_size_sampled(wls, irr, sh):
    """Handles whose tensor-core plan holds 13 and 11 MMA blocks (one CTA per SM, 512 TMEM columns)
    on the 1000-atom cell: sampled receivers against the oracle, computed one by one, and the
    status word clean."""
    wl = wls("diamond1k")
    conv = etp.EdgeConv(irr, sh, irr, 8, float(wl.r_cut))
    spec = ConvSpec(irr, sh, irr, 8, float(wl.r_cut))
    x, W, _ = _general_inputs(spec, wl.n_nodes, 79 + sh)
    g = _gpu_graph(wl)
    out = _np(conv.forward(g, torch.from_numpy(x).to(DEV), torch.from_numpy(W).to(DEV)))
    conv.check_status(DEV)
    rng = np.random.default_rng(19 + sh)
    sample = np.sort(rng.choice(wl.n_nodes, size=N_SAMPLE // 4, replace=False))
    ref, _ = forward_ref(wl, spec, x, W, sample=sample)
    assert_irrep_blocks_close(out[sample], ref, spec, "out", f"{irr} forward (sampled)")


@pytest.mark.parametrize("irin,sh,irout", GENERAL)
def test_general_irreps_weight_grad_parity(wls, irin, sh, irout):
    """dL/dW of general irreps handles against the oracle (small cell), and bitwise repeatable."""
    from oracle.conv import conv_vjp_weights
    wl = wls("tiny")
    conv = etp.EdgeConv(irin, sh, irout, 8, float(wl.r_cut))
    spec = ConvSpec(irin, sh, irout, 8, float(wl.r_cut))
    x, _, gout = _general_inputs(spec, wl.n_nodes, 3 * len(irin) + sh)
    g = _gpu_graph(wl)
    ref_g = full_graph(wl)
    xd, gd = torch.from_numpy(x).to(DEV), torch.from_numpy(gout).to(DEV)
    dW = conv.backward_weights(g, xd, gd)
    assert tuple(dW.shape) == (8, spec.weight_numel)
    ref = conv_vjp_weights(spec, ref_g["row_ptr"], ref_g["sender"], ref_g["edge_vec"], x, gout)
    ref = ref.reshape(8, spec.weight_numel)
    for p in range(len(spec.paths)):
        sl = spec.w_slice(p)
        assert_close_rel(_np(dW)[:, sl], ref[:, sl], f"{irin} dW path {p}")
    assert torch.equal(conv.backward_weights(g, xd, gd), dW)


def test_general_irreps_weight_grad_full_size(wls):
    """NequIP-L channel counts on the 1000-atom diamond cell: dL/dW against the oracle's weight VJP
    over the whole graph; as an extra, <dW, V> against the directional derivative <grad_out, F(V)>
    (exact: the output is linear in W), through the forward kernel."""
    from oracle.conv import conv_vjp_weights
    wl = wls("diamond1k")
    irr = "128x0e+64x1o+32x2e+32x3o"
    conv = etp.EdgeConv(irr, 3, irr, 8, float(wl.r_cut))
    spec = ConvSpec(irr, 3, irr, 8, float(wl.r_cut))
    x, W, gout = _general_inputs(spec, wl.n_nodes, 91)
    g = _gpu_graph(wl)
    xd, Wd, gd = (torch.from_numpy(a).to(DEV) for a in (x, W, gout))
    dW = conv.backward_weights(g, xd, gd).double()
    ref_g = full_graph(wl)
    ref = conv_vjp_weights(spec, ref_g["row_ptr"], ref_g["sender"], ref_g["edge_vec"], x, gout)
    assert_close_rel(_np(dW).reshape(ref.shape), ref, "NequIP-L diamond1k dL/dW vs oracle")
    dir_ = torch.from_numpy(np.random.default_rng(5).standard_normal(W.shape).astype(np.float32)).to(DEV)
    lhs = float((dW * dir_.double()).sum())
    rhs = float((conv.forward(g, xd, dir_).double() * gd.double()).sum())
    assert abs(lhs - rhs) <= 1e-4 * max(1.0, abs(rhs))


@pytest.mark.parametrize("irin,sh,irout", [("16x0e+16x1o+16x1e+16x2e+16x2o", 2, "16x0e+16x1o+16x1e+16x2e+16x2o"),
                                          ("128x0e+64x1o+32x2e+32x3o", 3, "128x0e+64x1o+32x2e+32x3o")])
def test_general_irreps_path_mask_parity(wls, irin, sh, irout, monkeypatch):
    """Per-edge path masks on general handles (at most 32 paths) against the oracle. Masked calls
    run the FP32 general forward, so with every bit set they equal its unmasked call bit for bit."""
    wl = wls("tiny")
    conv = etp.EdgeConv(irin, sh, irout, 8, float(wl.r_cut))
    spec = ConvSpec(irin, sh, irout, 8, float(wl.r_cut))
    x, W, gout = _general_inputs(spec, wl.n_nodes, 41)
    g = _gpu_graph(wl)
    ref_g = full_graph(wl)
    n_p = len(spec.paths)
    rng = np.random.default_rng(43)
    mask = rng.integers(0, 1 << n_p, size=g.n_edges).astype(np.int64)
    mask[: g.n_edges // 3] = (1 << n_p) - 1
    md = torch.from_numpy(mask.astype(np.uint32).view(np.int32)).to(DEV)
    xd, Wd, gd = (torch.from_numpy(a).to(DEV) for a in (x, W, gout))
    out = conv.forward(g, xd, Wd, path_mask=md)
    ref = conv_forward(spec, ref_g["row_ptr"], ref_g["sender"], ref_g["edge_vec"], x, W, path_mask=mask)
    assert_irrep_blocks_close(_np(out), ref, spec, "out", f"{irin} masked forward")
    gx, gv = conv.backward(g, xd, Wd, gd, path_mask=md)
    rgx, rgv = conv_vjp(spec, ref_g["row_ptr"], ref_g["sender"], ref_g["edge_vec"], x, W, gout, path_mask=mask)
    assert_irrep_blocks_close(_np(gx), rgx, spec, "in", f"{irin} masked grad_x")
    assert_close_rel(_np(gv), rgv, f"{irin} masked grad_edge_vec")
    # all bits set is the unmasked call of the same kernel, bit for bit
    ones = torch.full((g.n_edges,), -1, dtype=torch.int32, device=DEV)
    monkeypatch.setenv("ETP_GEN_FORWARD", "fp32")
    assert torch.equal(conv.forward(g, xd, Wd, path_mask=ones), conv.forward(g, xd, Wd))


def test_general_irreps_unsupported_calls_refuse(wls):
    wl = wls("tiny")
    irr = "32x0e+32x1o+32x2e+32x3o+32x4e"      # 42 paths: more than a 32-bit mask holds
    conv = etp.EdgeConv(irr, 4, irr, 8, float(wl.r_cut))
    spec = ConvSpec(irr, 4, irr, 8, float(wl.r_cut))
    x, W, gout = _general_inputs(spec, wl.n_nodes, 5)
    g = _gpu_graph(wl)
    xd, Wd, gd = (torch.from_numpy(a).to(DEV) for a in (x, W, gout))
    mask = torch.ones(g.n_edges, dtype=torch.int32, device=DEV)
    with pytest.raises(etp.EtpError) as ei:
        conv.forward(g, xd, Wd, path_mask=mask)
    assert ei.value.status == 3
    with pytest.raises(etp.EtpError) as ei:
        conv.radial_weights(g.edge_vec, Wd)
    assert ei.value.status == 3


def test_general_irreps_autograd_function(wls):
    """The autograd wrapper on a general handle: x, edge-vector and W gradients equal the ABI calls."""
    wl = wls("tiny")
    irr = "4x0e+3x1o+3x1e+4x2e"
    conv = etp.EdgeConv(irr, 2, irr, 8, float(wl.r_cut))
    spec = ConvSpec(irr, 2, irr, 8, float(wl.r_cut))
    x, W, gout = _general_inputs(spec, wl.n_nodes, 12)
    g = _gpu_graph(wl)
    fn = etp.edge_conv_function()
    xt = torch.from_numpy(x).to(DEV).requires_grad_(True)
    vt = g.edge_vec.clone().requires_grad_(True)
    Wt = torch.from_numpy(W).to(DEV).requires_grad_(True)
    gd = torch.from_numpy(gout).to(DEV)
    (fn.apply(conv, g, xt, vt, Wt) * gd).sum().backward()
    gx, gv = conv.backward(g, xt.detach(), Wt.detach(), gd)
    assert torch.equal(xt.grad, gx) and torch.equal(vt.grad, gv)
    assert torch.equal(Wt.grad, conv.backward_weights(g, xt.detach(), gd).reshape(Wt.shape))


# ------------------------------------------------------------------ full product ladder

@pytest.mark.parametrize("lmax,c,n,nu", [(2, 128, 4096, 3), (1, 32, 37, 2), (2, 64, 300, 3), (3, 32, 130, 2),
                                        (3, 96, 129, 3), (2, 128, 128, 1), (1, 128, 257, 4)])
def test_node_ladder_full_parity(lmax, c, n, nu):
    """The full ladder (per-rank path- and channel-mixing matrices on the tensor cores) against the
    oracle: the pages' 4096-node x 128-channel case and ragged tiles (node counts not a multiple of
    the 128-node tile), every rank and channel width; bitwise reproducible."""
    from oracle.product import full_step_sizes, node_ladder_full
    rng = np.random.default_rng(700 + 10 * lmax + nu + c)
    dim = (lmax + 1) ** 2 * c
    A = rng.standard_normal((n, dim)).astype(np.float32)
    steps = sum(full_step_sizes(lmax, c))
    assert etp.node_ladder_full_step_floats(lmax, c) == steps
    Ws = (rng.standard_normal((nu - 1, steps)) / np.sqrt(4 * c)).astype(np.float32)
    ref = node_ladder_full(lmax, c, A, list(Ws))
    Ad, Wd = torch.from_numpy(A).to(DEV), torch.from_numpy(Ws).to(DEV)
    out = etp.node_ladder_full(Ad, Wd, lmax)
    assert_blocks_close(_np(out), ref, c, lmax, f"full ladder lmax={lmax} C={c} N={n} nu={nu}")
    assert torch.equal(out, etp.node_ladder_full(Ad, Wd, lmax)), "full ladder is not bitwise deterministic"


def test_node_ladder_full_with_diagonal_matrices_matches_the_path_reduced_kernel():
    """Channel-diagonal matrices make the full ladder the path-reduced one: the two kernels agree."""
    from oracle.product import paths_of_rank
    lmax, c, n, nu = 2, 64, 500, 3
    rng = np.random.default_rng(77)
    A = rng.standard_normal((n, 9 * c)).astype(np.float32)
    wr = (rng.standard_normal((nu - 1, len(product_paths_of(lmax)), c)) / 2).astype(np.float32)
    full = []
    for q in range(nu - 1):
        blocks = []
        for l3 in range(lmax + 1):
            ps = paths_of_rank(lmax, l3)
            m = np.zeros((c, len(ps) * c), np.float32)
            for j, p in enumerate(ps):
                m[np.arange(c), j * c + np.arange(c)] = wr[q, p]
            blocks.append(m.ravel())
        full.append(np.concatenate(blocks))
    Ad = torch.from_numpy(A).to(DEV)
    got = etp.node_ladder_full(Ad, torch.from_numpy(np.stack(full)).to(DEV), lmax)
    red = etp.node_ladder(Ad, torch.from_numpy(wr).to(DEV), lmax)
    assert_blocks_close(_np(got), _np(red).astype(np.float64), c, lmax, "full ladder with diagonal matrices")


def product_paths_of(lmax):
    from oracle.product import product_paths
    return product_paths(lmax)
