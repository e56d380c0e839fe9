"""C-ABI checks that need no GPU: the library loads, exports every declared symbol, and its
host-side logic (irreps parsing, path enumeration, argument checks) behaves as documented."""
import ctypes
import os
import re

import numpy as np
import pytest

import equivariant_mlip_tensor_edge_b200 as etp
from oracle.conv import ConvSpec, flop_counts

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "etp.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(etp_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    return etp.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert len(names) >= 13
    for n in names:
        assert hasattr(lib, n), n
        assert n in etp.SIGNATURES, f"{n} has no ctypes signature in the binding"


def _create(irin, lmax, irout, nb=8, rc=5.0):
    lib = etp.load_library()
    h = ctypes.c_void_p()
    st = lib.etp_create(irin.encode() if irin is not None else None, lmax,
                        irout.encode() if irout is not None else None, nb, rc, ctypes.byref(h))
    if st == 0:
        lib.etp_destroy(h)
    return st


def test_create_status_codes():
    assert _create("64x0e+64x1o+64x2e", 2, "64x0e+64x1o+64x2e") == 0
    assert _create("8x0e + 8x1o", 1, "8x0e+8x1o") == 0
    assert _create("64x0e+64x1q", 1, "64x0e+64x1o") == 2        # malformed
    assert _create("64x0e++64x1o", 1, "64x0e+64x1o") == 2
    assert _create(None, 1, "64x0e+64x1o") == 2
    # general handles (table-driven kernels)
    assert _create("64x0e+64x1e", 1, "64x0e+64x1e") == 0        # parity not (-1)^l
    assert _create("64x0e+32x1o", 1, "64x0e+32x1o") == 0        # mixed multiplicity
    assert _create("6x0e+6x1o", 1, "6x0e+6x1o") == 0            # C % 4 != 0
    assert _create("8x0e+8x1o", 2, "8x0e+8x1o") == 0            # sh_lmax != L
    assert _create("8x0e+8x1o+8x2e+8x3o+8x4e", 4, "8x0e+8x1o+8x2e+8x3o+8x4e") == 0
    # outside both
    assert _create("8x0e+8x1o", 1, "8x0e+8x1o", nb=6) == 3      # n_basis != 8
    assert _create("8x0e+8x5o", 1, "8x0e+8x5o") == 3            # l > 4
    assert _create("8x0e+8x1o", 5, "8x0e+8x1o") == 3            # sh_lmax > 4
    assert _create("8x0e", 0, "4x0e") == 3                      # no path (multiplicities differ)
    assert _create("1024x0e+1024x1o+1024x2e", 2, "1024x0e+1024x1o+1024x2e") == 3   # rows above 4096 floats
    assert _create("8x0e+8x1o", 1, "8x0e+8x1o", rc=-1.0) == 1


@pytest.mark.parametrize("lmax,c", [(1, 8), (2, 64), (3, 128)])
def test_info_matches_independent_path_enumeration(lmax, c):
    irr = "+".join(f"{c}x{l}{'eo'[l % 2]}" for l in range(lmax + 1))
    conv = etp.EdgeConv(irr, lmax, irr, 8, 5.0)
    spec = ConvSpec(irr, lmax, irr, 8, 5.0)
    fc = flop_counts(spec)
    assert conv.info["n_paths"] == len(spec.paths)
    assert conv.info["cg_nnz"] == fc["nnz"]
    assert conv.info["sum_2l3p1"] == fc["sum_2l3p1"]
    assert conv.info["dim_in"] == spec.dim_in == conv.info["dim_out"]
    assert conv.info["weight_numel"] == 8 * len(spec.paths) * c
    assert conv.info["flop_fwd"] == fc["fwd_tp"] and conv.info["flop_bwd"] == fc["bwd_tp"]
    assert conv.paths == [tuple(p) for p in spec.paths]
    buf = (ctypes.c_int * 3)()
    assert etp.load_library().etp_get_paths(conv._h, buf, 1) == 6    # capacity below n_paths
    assert conv.workspace_bytes(100, 1000) >= 2 * 4 * 1000


@pytest.mark.parametrize("irin,sh,irout", [
    ("4x0e+3x1o+3x1e+4x2e+2x2o+3x3o+4x4e", 4, "4x0e+3x1o+3x1e+4x2e+2x2o+3x3o+4x4e"),
    ("128x0e+64x1o+32x2e+32x3o", 3, "128x0e+64x1o+32x2e+32x3o"),
    ("16x0e+16x1o", 2, "16x0e+16x1o+16x1e+16x2e"),
    ("6x0e+6x1o+6x2e", 2, "6x0e+6x1o+6x2e"),
])
def test_general_info_matches_independent_path_enumeration(irin, sh, irout):
    conv = etp.EdgeConv(irin, sh, irout, 8, 5.0)
    spec = ConvSpec(irin, sh, irout, 8, 5.0)
    fc = flop_counts(spec)
    assert conv.info["general"] == 1
    assert conv.info["n_paths"] == len(spec.paths)
    assert conv.info["cg_nnz"] == fc["nnz"]
    assert conv.info["sum_2l3p1"] == fc["sum_2l3p1"]
    assert conv.info["dim_in"] == spec.dim_in and conv.info["dim_out"] == spec.dim_out
    assert conv.info["weight_numel"] == 8 * spec.weight_numel
    assert conv.info["channels"] == (spec.channels or 0)
    assert conv.info["flop_fwd"] == fc["fwd_tp"] and conv.info["flop_bwd"] == fc["bwd_tp"]
    assert conv.paths == [tuple(p) for p in spec.paths]
    assert etp.EdgeConv("8x0e+8x1o", 1, "8x0e+8x1o", 8, 5.0).info["general"] == 0


def test_status_strings_and_errors(lib):
    for s in range(7):
        assert lib.etp_status_string(s)
    with pytest.raises(etp.EtpError) as ei:
        etp.EdgeConv("8x0e+8x1o", 1, "8x0e+8x5o", 8, 5.0)
    assert ei.value.status == 3
    assert "etp_create" in str(ei.value)


def test_null_arguments_rejected_without_cuda(lib):
    # argument checks happen on the host before any CUDA call
    conv = etp.EdgeConv("8x0e+8x1o", 1, "8x0e+8x1o", 8, 4.0)
    st = lib.etp_forward(conv._h, 10, 5, None, None, None, None, None, None, None, 0, None)
    assert st == 1
    st = lib.etp_forward(None, 10, 5, None, None, None, None, None, None, None, 0, None)
    assert st == 1
    st = lib.etp_backward(conv._h, 10, 5, None, None, None, None, None, None, None, None, None, None, None, 0, None)
    assert st == 1
    assert lib.etp_forces(-1, 0, None, None, None, None, None, None) == 1
    assert lib.etp_neighbors(None, -1, None, None, 1.0, 0, None, None, None, None, None, None, None, None, 0,
                             None) == 1


def test_general_workspace_covers_every_scratch():
    """General handles: receiver map + validation scratch + the larger of the edge-gradient shares
    (3 floats per edge and input block) and the weight gradient's partial columns (8 x cols per
    range of 128 edges)."""
    irr = "128x0e+64x1o+32x2e+32x3o"
    conv = etp.EdgeConv(irr, 3, irr, 8, 5.0)
    spec = ConvSpec(irr, 3, irr, 8, 5.0)
    for n_nodes, n_edges in ((10, 0), (1000, 89156), (5, 129)):
        nb = conv.workspace_bytes(n_nodes, n_edges)
        in_blocks = len({bi for bi, _, _ in spec.paths})
        ranges = max(1, -(-n_edges // 128))
        need = 4 * n_edges + 4 * (n_edges + 1) + max(12 * n_edges * in_blocks if in_blocks > 1 else 0,
                                                       4 * 8 * spec.weight_numel * ranges)
        assert nb >= need, (n_nodes, n_edges, nb, need)


def _irreps_str(blocks):
    return "+".join(f"{m}x{l}{'e' if p > 0 else 'o'}" for m, l, p in blocks)


def test_create_matches_the_oracle_path_set_on_random_irreps():
    """etp_create on random irreps strings (seeded): when the oracle finds paths and the sizes fit,
    the handle exists and its path list, dimensions and weight columns equal the oracle's; otherwise
    the call is refused as unsupported. No other outcome."""
    rng = np.random.default_rng(2024)
    lib = etp.load_library()
    seen_general = seen_uniform = seen_refused = 0
    for _ in range(300):
        def blocks():
            k = int(rng.integers(1, 6))
            return [(int(rng.choice([1, 3, 4, 8, 16, 32])), int(rng.integers(0, 5)), int(rng.choice([1, -1])))
                    for _ in range(k)]
        bin_, bout = blocks(), (blocks() if rng.random() < 0.5 else None)
        bout = bout if bout is not None else list(bin_)
        sh = int(rng.integers(0, 5))
        irin, irout = _irreps_str(bin_), _irreps_str(bout)
        spec = ConvSpec(irin, sh, irout, 8, 5.0)
        h = ctypes.c_void_p()
        st = lib.etp_create(irin.encode(), sh, irout.encode(), 8, 5.0, ctypes.byref(h))
        fits = (len(spec.paths) >= 1 and len(spec.paths) <= 128 and spec.dim_in <= 4096 and spec.dim_out <= 4096
                and len(bin_) <= 16 and len(bout) <= 16)
        if not fits:
            assert st == 3, (irin, sh, irout, st)
            seen_refused += 1
            continue
        assert st == 0, (irin, sh, irout, st, lib.etp_last_error())
        info = etp.EtpInfo()
        assert lib.etp_get_info(h, ctypes.byref(info)) == 0
        buf = (ctypes.c_int * (3 * len(spec.paths)))()
        assert lib.etp_get_paths(h, buf, len(spec.paths)) == 0
        got = [tuple(buf[3 * p:3 * p + 3]) for p in range(len(spec.paths))]
        assert got == [tuple(p) for p in spec.paths]
        assert (info.dim_in, info.dim_out, info.n_paths) == (spec.dim_in, spec.dim_out, len(spec.paths))
        assert info.weight_numel == 8 * spec.weight_numel
        seen_general += info.general
        seen_uniform += 1 - info.general
        lib.etp_destroy(h)
    assert seen_general > 50 and seen_refused > 5


def test_status_word_gates_calls_until_get_status_clears_it(lib):
    """A kernel that gives up a bounded wait stores its code in the handle's status word; every
    later compute call on the handle then fails with ETP_ERR_CUDA (before any CUDA work) until
    etp_get_status has read and cleared the word. Here the test writes the word itself."""
    conv = etp.EdgeConv("8x0e+8x1o", 1, "8x0e+8x1o", 8, 4.0)
    word = lib.etp_status_word(conv._h)
    assert word and word[0] == 0
    assert not lib.etp_status_word(None)
    # a clean handle: radial weights of an empty edge list is a no-op that succeeds
    assert lib.etp_radial_weights(conv._h, 0, None, None, None, None) == 0
    word[0] = 37
    fake = ctypes.c_void_p(0x1000)   # 16-byte aligned, never dereferenced: the gate comes first
    assert lib.etp_forward(conv._h, 4, 4, fake, fake, fake, fake, fake, fake, fake, 1 << 20, None) == 5
    assert "code 37" in lib.etp_last_error().decode()
    assert lib.etp_forward_noalloc(conv._h, 4, 4, fake, fake, fake, fake, fake, fake, None) == 5
    assert lib.etp_backward_weights(conv._h, 4, 4, fake, fake, fake, fake, fake, fake, fake, 1 << 20, None) == 5
    assert lib.etp_radial_weights(conv._h, 0, None, None, None, None) == 5
    code = ctypes.c_int(-1)
    assert lib.etp_get_status(conv._h, None, ctypes.byref(code)) == 5
    assert code.value == 37
    assert word[0] == 0
    assert lib.etp_get_status(conv._h, None, ctypes.byref(code)) == 0 and code.value == 0
    assert lib.etp_radial_weights(conv._h, 0, None, None, None, None) == 0
    assert lib.etp_get_status(None, None, None) == 1
    # the binding raises on a set word
    word[0] = 12
    with pytest.raises(etp.EtpError) as ei:
        conv.check_status()
    assert ei.value.status == 5 and "code 12" in str(ei.value)
    conv.check_status()


def test_node_ladder_full_refuses_unsupported_shapes_before_device_work():
    """Widths other than 32, 64, 96, 128, ranks outside 1..3, orders outside 1..8 and a missing
    workspace are refused by the host checks, before any device pointer is touched."""
    import equivariant_mlip_tensor_edge_b200 as etp
    lib = etp.load_library()
    fake = ctypes.c_void_p(256)
    assert lib.etp_node_ladder_full(2, 16, 10, 2, fake, fake, fake, fake, 1 << 30, None) == 3   # ETP_ERR_UNSUPPORTED
    assert lib.etp_node_ladder_full(4, 32, 10, 2, fake, fake, fake, fake, 1 << 30, None) == 3
    assert lib.etp_node_ladder_full(2, 32, 10, 9, fake, fake, fake, fake, 1 << 30, None) == 1   # ETP_ERR_INVALID_ARG
    assert lib.etp_node_ladder_full(2, 32, 10, 2, fake, fake, fake, None, 0, None) == 1
    assert lib.etp_node_ladder_full_step_floats(2, 32) == 11 * 32 * 32
    assert lib.etp_node_ladder_full_workspace_bytes(2, 16, 10) == 0
