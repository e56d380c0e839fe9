"""etp_forward_noalloc: the forward whose scratch is a fixed array of the library's device module.

Called through the C ABI and compared with etp_forward (which takes a caller workspace) on the
same inputs, on two calls in a row, at the parity tolerance. The file name keeps it last in
collection, so it also runs after every other test has used the library.
"""
import ctypes

import numpy as np
import pytest

import equivariant_mlip_tensor_edge_b200 as etp
import workloads
from tests._oracle_side import assert_blocks_close
from oracle.conv import ConvSpec, conv_forward

ETP_ERR_CAPACITY = 6


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc(conv, g, x, W, out, stream):
    lib = etp.load_library()
    return lib.etp_forward_noalloc(conv._h, g.n_nodes, g.n_edges, _ptr(g.row_ptr), _ptr(g.sender),
                                   _ptr(g.edge_vec), _ptr(x), _ptr(W), _ptr(out), ctypes.c_void_p(stream))


def _check_two_calls(conv, g, x, W, channels, lmax, what, oracle_ref=None):
    """Two no-alloc calls in a row against etp_forward and, when given, against the oracle."""
    import torch
    ref = conv.forward(g, x, W)
    if oracle_ref is not None:
        assert_blocks_close(ref.cpu().numpy().astype(np.float64), oracle_ref, channels, lmax,
                            f"{what}: etp_forward vs oracle")
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        st = _noalloc(conv, g, x, W, out, stream)
        assert st == 0, etp.load_library().etp_last_error().decode()
        torch.cuda.synchronize()
        got = out.cpu().numpy().astype(np.float64)
        assert_blocks_close(got, ref.cpu().numpy().astype(np.float64), channels, lmax,
                            f"{what}: no-alloc call {call + 1} vs etp_forward")
        if oracle_ref is not None:
            assert_blocks_close(got, oracle_ref, channels, lmax, f"{what}: no-alloc call {call + 1} vs oracle")


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["tiny", "diamond1k"])
def test_noalloc_forward_matches_workspace_forward(name):
    import torch
    wl = workloads.make(name)
    conv = etp.EdgeConv(wl.irreps, wl.lmax, wl.irreps, wl.n_basis, float(wl.r_cut))
    g = etp.neighbors(torch.from_numpy(wl.pos).to("cuda"), float(wl.r_cut), cell=wl.cell, pbc=wl.pbc)
    x = torch.from_numpy(wl.features()).to("cuda")
    W = torch.from_numpy(wl.weights(conv.n_paths)).to("cuda")
    _check_two_calls(conv, g, x, W, wl.channels, wl.lmax, name)


@pytest.mark.gpu
def test_noalloc_forward_lmax3_largest_accepted_channels():
    """lmax 3 with 160 channels: the largest scratch that fits the fixed array. Both etp_forward and
    the no-alloc entry are compared with the oracle on this ragged graph (degrees 0..69)."""
    import torch
    c, lmax, n = 160, 3, 40
    irr = "+".join(f"{c}x{l}{'eo'[l % 2]}" for l in range(lmax + 1))
    conv = etp.EdgeConv(irr, lmax, irr, 8, 5.0)
    rng = np.random.default_rng(7)
    degrees = rng.integers(0, 70, size=n)
    recv = np.repeat(np.arange(n), degrees)
    send = rng.integers(0, n, size=len(recv))
    d = rng.standard_normal((len(recv), 3))
    vec = (d / np.linalg.norm(d, axis=1, keepdims=True) * rng.uniform(0.5, 4.5, (len(recv), 1))).astype(np.float32)
    g = etp.build_csr(n, torch.from_numpy(recv).to("cuda"), torch.from_numpy(send).to("cuda"),
                      torch.from_numpy(vec).to("cuda"))
    x = torch.from_numpy(rng.standard_normal((n, conv.info["dim_in"])).astype(np.float32)).to("cuda")
    W = torch.from_numpy((rng.standard_normal((8, conv.n_paths, c)) / np.sqrt(8)).astype(np.float32)).to("cuda")
    spec = ConvSpec(irr, lmax, irr, 8, 5.0)
    row_ptr = np.concatenate([[0], np.cumsum(degrees)])
    oracle_ref = conv_forward(spec, row_ptr, send, vec, x.cpu().numpy(), W.cpu().numpy())
    _check_two_calls(conv, g, x, W, c, lmax, "lmax3 C160", oracle_ref=oracle_ref)


def test_noalloc_forward_refuses_scratch_beyond_the_fixed_array():
    """lmax 3 with 192 channels needs more than 256 KiB: refused before any device work."""
    lib = etp.load_library()
    irr = "192x0e+192x1o+192x2e+192x3o"
    conv = etp.EdgeConv(irr, 3, irr, 8, 5.0)
    fake = ctypes.c_void_p(256)       # never dereferenced: the size check comes first
    st = lib.etp_forward_noalloc(conv._h, 10, 20, fake, fake, fake, fake, fake, fake, None)
    assert st == ETP_ERR_CAPACITY
    msg = lib.etp_last_error().decode()
    assert "262144" in msg and "etp_forward" in msg
