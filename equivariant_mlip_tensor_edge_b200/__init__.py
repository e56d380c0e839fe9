"""B200-native equivariant edge tensor-product convolution: Python binding of libetp.so.

Argument marshalling only. Every step of the path (neighbour list, CSR, spherical harmonics,
radial basis and projection, Clebsch-Gordan contraction, segmented sums, backward, forces)
runs in the CUDA kernels of ``libetp.so``; PyTorch provides device memory and streams. There
is no CPU fallback: without the built library, or without a CUDA device, calls raise.

The C ABI is documented in ``include/etp.h``.
"""
import ctypes
import os
from dataclasses import dataclass

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libetp.so")

ETP_OK = 0
STATUS_NAMES = {0: "ETP_OK", 1: "ETP_ERR_INVALID_ARG", 2: "ETP_ERR_IRREPS", 3: "ETP_ERR_UNSUPPORTED",
                4: "ETP_ERR_BAD_GRAPH", 5: "ETP_ERR_CUDA", 6: "ETP_ERR_CAPACITY"}

# exported symbols and their C signatures (restype, argtypes)
_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_ip = ctypes.POINTER(ctypes.c_int)
_dp = ctypes.POINTER(ctypes.c_double)


class EtpInfo(ctypes.Structure):
    _fields_ = [("lmax", ctypes.c_int), ("channels", ctypes.c_int), ("dim_in", ctypes.c_int),
                ("dim_out", ctypes.c_int), ("n_paths", ctypes.c_int), ("n_basis", ctypes.c_int),
                ("weight_numel", ctypes.c_int), ("cg_nnz", ctypes.c_int), ("sum_2l3p1", ctypes.c_int),
                ("r_cut", ctypes.c_float), ("general", ctypes.c_int), ("flop_fwd", ctypes.c_int),
                ("flop_bwd", ctypes.c_int)]


SIGNATURES = {
    "etp_create": (_i, [ctypes.c_char_p, _i, ctypes.c_char_p, _i, _f, ctypes.POINTER(_vp)]),
    "etp_destroy": (_i, [_vp]),
    "etp_get_info": (_i, [_vp, ctypes.POINTER(EtpInfo)]),
    "etp_get_paths": (_i, [_vp, _ip, _i]),
    "etp_status_string": (ctypes.c_char_p, [_i]),
    "etp_last_error": (ctypes.c_char_p, []),
    "etp_workspace_bytes": (_sz, [_vp, _i, _i]),
    "etp_forward": (_i, [_vp, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "etp_forward_noalloc": (_i, [_vp, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "etp_backward": (_i, [_vp, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "etp_backward_weights": (_i, [_vp, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "etp_forward_masked": (_i, [_vp, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "etp_backward_masked": (_i, [_vp, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                                 _vp]),
    "etp_radial_weights": (_i, [_vp, _i, _vp, _vp, _vp, _vp]),
    "etp_node_ladder": (_i, [_i, _i, _i, _i, _vp, _vp, _vp, _vp]),
    "etp_node_ladder_full_step_floats": (_sz, [_i, _i]),
    "etp_node_ladder_full_workspace_bytes": (_sz, [_i, _i, _i]),
    "etp_node_ladder_full": (_i, [_i, _i, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
    "etp_forces": (_i, [_i, _i, _vp, _vp, _vp, _vp, _vp, _vp]),
    "etp_graph_workspace_bytes": (_sz, [_i, _i]),
    "etp_neighbors": (_i, [_vp, _i, _dp, _ip, _f, _i, _ip, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "etp_build_csr": (_i, [_i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "etp_get_status": (_i, [_vp, _vp, _ip]),
    "etp_status_word": (_ip, [_vp]),
}

_lib = None


def load_library(path=LIB_PATH):
    """Load libetp.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with `python -m equivariant_mlip_tensor_edge_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class EtpError(RuntimeError):
    def __init__(self, status, where):
        lib = load_library()
        msg = lib.etp_last_error().decode()
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def _check(status, where):
    if status != ETP_OK:
        raise EtpError(status, where)


def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    torch = _torch()
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need_cuda(*tensors):
    for t in tensors:
        if t is not None and not t.is_cuda:
            raise ValueError("libetp operates on CUDA tensors only (no CPU fallback)")


def _i32(t):
    torch = _torch()
    return t if t.dtype == torch.int32 and t.is_contiguous() else t.to(torch.int32).contiguous()


def _f32(t):
    torch = _torch()
    return t if t.dtype == torch.float32 and t.is_contiguous() else t.to(torch.float32).contiguous()


@dataclass
class Graph:
    """Receiver-sorted CSR edge layout plus the transposed (sender-sorted) order (device tensors)."""
    n_nodes: int
    n_edges: int
    row_ptr: object
    sender: object
    edge_vec: object
    t_row_ptr: object
    t_perm: object
    shift: object = None
    perm: object = None


def graph_workspace_bytes(n_nodes, max_edges):
    return load_library().etp_graph_workspace_bytes(n_nodes, max_edges)


def neighbors(pos, r_cut, cell=None, pbc=(False, False, False), max_edges=None, with_shift=True):
    """Neighbour list + canonical CSR on the GPU. pos: [N,3] float32 CUDA tensor; cell: 3x3 (host)."""
    torch = _torch()
    lib = load_library()
    _need_cuda(pos)
    pos = _f32(pos)
    n = pos.shape[0]
    dev = pos.device
    if max_edges is None:
        max_edges = max(1024, n * 128)
    cell_arr = None
    if cell is not None:
        vals = [float(v) for row in cell for v in row]
        cell_arr = (ctypes.c_double * 9)(*vals)
    pbc_arr = (ctypes.c_int * 3)(*[int(bool(p)) for p in pbc])
    while True:
        row_ptr = torch.empty(n + 1, dtype=torch.int32, device=dev)
        t_row_ptr = torch.empty(n + 1, dtype=torch.int32, device=dev)
        sender = torch.empty(max(max_edges, 1), dtype=torch.int32, device=dev)
        edge_vec = torch.empty((max(max_edges, 1), 3), dtype=torch.float32, device=dev)
        shift = torch.empty((max(max_edges, 1), 3), dtype=torch.int32, device=dev) if with_shift else None
        t_perm = torch.empty(max(max_edges, 1), dtype=torch.int32, device=dev)
        ws_bytes = lib.etp_graph_workspace_bytes(n, max_edges)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        n_edges = ctypes.c_int(0)
        st = lib.etp_neighbors(_ptr(pos), n, ctypes.cast(cell_arr, _dp) if cell_arr is not None else None, pbc_arr,
                               float(r_cut), max_edges, ctypes.byref(n_edges), _ptr(row_ptr), _ptr(sender),
                               _ptr(edge_vec), _ptr(shift), _ptr(t_row_ptr), _ptr(t_perm), _ptr(ws), ws_bytes,
                               _stream(dev))
        if st == 6:  # capacity: retry with the reported count
            max_edges = n_edges.value
            continue
        _check(st, "etp_neighbors")
        e = n_edges.value
        return Graph(n, e, row_ptr, sender[:e], edge_vec[:e], t_row_ptr, t_perm[:e],
                     shift[:e] if shift is not None else None)


def build_csr(n_nodes, receiver, sender, edge_vec):
    """Canonical CSR of a given edge list (any order), on the GPU."""
    torch = _torch()
    lib = load_library()
    _need_cuda(receiver, sender, edge_vec)
    receiver, sender, edge_vec = _i32(receiver), _i32(sender), _f32(edge_vec)
    e = receiver.shape[0]
    dev = receiver.device
    row_ptr = torch.empty(n_nodes + 1, dtype=torch.int32, device=dev)
    t_row_ptr = torch.empty(n_nodes + 1, dtype=torch.int32, device=dev)
    s_out = torch.empty(max(e, 1), dtype=torch.int32, device=dev)
    v_out = torch.empty((max(e, 1), 3), dtype=torch.float32, device=dev)
    perm = torch.empty(max(e, 1), dtype=torch.int32, device=dev)
    t_perm = torch.empty(max(e, 1), dtype=torch.int32, device=dev)
    ws_bytes = lib.etp_graph_workspace_bytes(n_nodes, e)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    _check(lib.etp_build_csr(n_nodes, e, _ptr(receiver), _ptr(sender), _ptr(edge_vec), _ptr(row_ptr),
                             _ptr(s_out), _ptr(v_out), _ptr(perm), _ptr(t_row_ptr), _ptr(t_perm), _ptr(ws),
                             ws_bytes, _stream(dev)), "etp_build_csr")
    return Graph(n_nodes, e, row_ptr, s_out[:e], v_out[:e], t_row_ptr, t_perm[:e], None, perm[:e])


def forces(graph, grad_edge_vec, out=None):
    torch = _torch()
    lib = load_library()
    _need_cuda(grad_edge_vec)
    if out is None:
        out = torch.empty((graph.n_nodes, 3), dtype=torch.float32, device=grad_edge_vec.device)
    _check(lib.etp_forces(graph.n_nodes, graph.n_edges, _ptr(graph.row_ptr), _ptr(graph.t_row_ptr),
                          _ptr(graph.t_perm), _ptr(_f32(grad_edge_vec)), _ptr(out), _stream(out.device)),
           "etp_forces")
    return out


class EdgeConv:
    """Handle for one convolution configuration (irreps, SH lmax, radial basis, cutoff).

    Uniform irreps (C x (0e + 1o + ... + Le), SH lmax L <= 3) run on the tensor-core kernels;
    anything else the library supports (per-block multiplicities, both parities, rank <= 4) on the
    general kernels (``info["general"] == 1``), whose W is [n_basis, cols] in ``paths`` order.
    """

    def __init__(self, irreps_in, sh_lmax, irreps_out, n_basis=8, r_cut=5.0):
        lib = load_library()
        h = ctypes.c_void_p()
        _check(lib.etp_create(irreps_in.encode(), int(sh_lmax), irreps_out.encode(), int(n_basis),
                              float(r_cut), ctypes.byref(h)), "etp_create")
        self._h = h
        info = EtpInfo()
        _check(lib.etp_get_info(h, ctypes.byref(info)), "etp_get_info")
        self.info = {k: getattr(info, k) for k, _ in EtpInfo._fields_}
        self.r_cut = float(r_cut)

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and _lib is not None:
            _lib.etp_destroy(h)
            self._h = None

    @property
    def n_paths(self):
        return self.info["n_paths"]

    @property
    def paths(self):
        """[(input block, l2, output block)] in W's column order."""
        n = self.n_paths
        buf = (ctypes.c_int * (3 * n))()
        _check(load_library().etp_get_paths(self._h, buf, n), "etp_get_paths")
        return [tuple(buf[3 * p:3 * p + 3]) for p in range(n)]

    def workspace_bytes(self, n_nodes, n_edges):
        return load_library().etp_workspace_bytes(self._h, n_nodes, n_edges)

    def check_status(self, device=None):
        """Synchronise the current stream and raise if a kernel of an earlier call on this handle
        gave up a bounded pipeline wait (the code is cleared)."""
        code = ctypes.c_int(0)
        stream = _stream(device) if device is not None else None
        _check(load_library().etp_get_status(self._h, stream, ctypes.byref(code)), "etp_get_status")

    def _workspace(self, n_nodes, n_edges, device, workspace):
        torch = _torch()
        nb = self.workspace_bytes(n_nodes, n_edges)
        if workspace is None or workspace.numel() < nb:
            workspace = torch.empty(max(nb, 1), dtype=torch.uint8, device=device)
        return workspace, nb

    def forward(self, graph, x, W, out=None, workspace=None, path_mask=None):
        """path_mask: optional int32 CUDA tensor [n_edges] (canonical order), bit p = path p on."""
        torch = _torch()
        _need_cuda(x, W, graph.row_ptr)
        x, W = _f32(x), _f32(W)
        if out is None:
            out = torch.empty((graph.n_nodes, self.info["dim_out"]), dtype=torch.float32, device=x.device)
        ws, nb = self._workspace(graph.n_nodes, graph.n_edges, x.device, workspace)
        lib = load_library()
        if path_mask is None:
            _check(lib.etp_forward(self._h, graph.n_nodes, graph.n_edges, _ptr(graph.row_ptr),
                                   _ptr(graph.sender), _ptr(graph.edge_vec), _ptr(x), _ptr(W), _ptr(out),
                                   _ptr(ws), nb, _stream(x.device)), "etp_forward")
        else:
            _need_cuda(path_mask)
            m = _i32(path_mask)
            _check(lib.etp_forward_masked(self._h, graph.n_nodes, graph.n_edges, _ptr(graph.row_ptr),
                                          _ptr(graph.sender), _ptr(graph.edge_vec), _ptr(x), _ptr(W), _ptr(m),
                                          _ptr(out), _ptr(ws), nb, _stream(x.device)), "etp_forward_masked")
        return out

    def backward(self, graph, x, W, grad_out, want_grad_x=True, want_grad_vec=True, grad_x=None,
                 grad_vec=None, workspace=None, path_mask=None):
        torch = _torch()
        _need_cuda(x, W, grad_out)
        x, W, grad_out = _f32(x), _f32(W), _f32(grad_out)
        dev = x.device
        if want_grad_x and grad_x is None:
            grad_x = torch.empty((graph.n_nodes, self.info["dim_in"]), dtype=torch.float32, device=dev)
        if want_grad_vec and grad_vec is None:
            grad_vec = torch.empty((max(graph.n_edges, 1), 3), dtype=torch.float32, device=dev)[:graph.n_edges]
        ws, nb = self._workspace(graph.n_nodes, graph.n_edges, dev, workspace)
        gx_p = _ptr(grad_x) if want_grad_x else None
        gv_p = _ptr(grad_vec) if want_grad_vec else None
        if path_mask is None:
            _check(load_library().etp_backward(
                self._h, graph.n_nodes, graph.n_edges, _ptr(graph.row_ptr), _ptr(graph.sender), _ptr(graph.edge_vec),
                _ptr(graph.t_row_ptr), _ptr(graph.t_perm), _ptr(x), _ptr(W), _ptr(grad_out), gx_p, gv_p, _ptr(ws), nb,
                _stream(dev)), "etp_backward")
        else:
            _need_cuda(path_mask)
            m = _i32(path_mask)
            _check(load_library().etp_backward_masked(
                self._h, graph.n_nodes, graph.n_edges, _ptr(graph.row_ptr), _ptr(graph.sender), _ptr(graph.edge_vec),
                _ptr(graph.t_row_ptr), _ptr(graph.t_perm), _ptr(x), _ptr(W), _ptr(m), _ptr(grad_out), gx_p, gv_p,
                _ptr(ws), nb, _stream(dev)), "etp_backward_masked")
        return (grad_x if want_grad_x else None), (grad_vec if want_grad_vec else None)

    def backward_weights(self, graph, x, grad_out, grad_W=None, workspace=None):
        """dL/dW for L = <grad_out, forward(graph, x, W)>: [n_basis, n_paths, C], or [n_basis, cols] for
        a general irreps handle."""
        torch = _torch()
        _need_cuda(x, grad_out)
        x, grad_out = _f32(x), _f32(grad_out)
        if grad_W is None:
            shape = ((self.info["n_basis"], self.info["n_paths"], self.info["channels"]) if not self.info["general"]
                     else (self.info["n_basis"], self.info["weight_numel"] // self.info["n_basis"]))
            grad_W = torch.empty(shape, dtype=torch.float32, device=x.device)
        ws, nb = self._workspace(graph.n_nodes, graph.n_edges, x.device, workspace)
        _check(load_library().etp_backward_weights(
            self._h, graph.n_nodes, graph.n_edges, _ptr(graph.row_ptr), _ptr(graph.sender), _ptr(graph.edge_vec),
            _ptr(x), _ptr(grad_out), _ptr(grad_W), _ptr(ws), nb, _stream(x.device)), "etp_backward_weights")
        return grad_W

    def radial_weights(self, edge_vec, W):
        torch = _torch()
        _need_cuda(edge_vec, W)
        edge_vec, W = _f32(edge_vec), _f32(W)
        e = edge_vec.shape[0]
        out = torch.empty((max(e, 1), self.n_paths, self.info["channels"]), dtype=torch.float32,
                          device=edge_vec.device)[:e]
        _check(load_library().etp_radial_weights(self._h, e, _ptr(edge_vec), _ptr(W), _ptr(out),
                                                 _stream(edge_vec.device)), "etp_radial_weights")
        return out


def node_ladder(A, Ws, lmax, out=None):
    """Node-local product ladder: out = B_1 + ... + B_nu with B_1 = A and B_{q+1} = P(B_q, A; Ws[q-1]).

    A: [N, C (lmax+1)^2] float32 CUDA tensor (node-row layout); Ws: [nu - 1, n_paths, C] (nu - 1 may
    be 0). Returns out like A.
    """
    torch = _torch()
    _need_cuda(A, Ws)
    A, Ws = _f32(A), _f32(Ws)
    n, dim = A.shape
    c = dim // ((lmax + 1) ** 2)
    nu = Ws.shape[0] + 1
    if out is None:
        out = torch.empty_like(A)
    _check(load_library().etp_node_ladder(int(lmax), c, n, nu, _ptr(A), _ptr(Ws) if nu > 1 else None, _ptr(out),
                                          _stream(A.device)), "etp_node_ladder")
    return out


def node_ladder_full_step_floats(lmax, channels):
    """Floats of one step of full-ladder weights (the per-rank matrices [C][P_l3 C], l3 = 0..lmax)."""
    return int(load_library().etp_node_ladder_full_step_floats(int(lmax), int(channels)))


def node_ladder_full(A, Ws, lmax, out=None, workspace=None):
    """The full product ladder: out = B_1 + ... + B_nu, B_1 = A, and each step the per-path products
    of B_q and A compressed by that step's per-rank matrices (paths and channels mixed; the mixing
    runs on the tensor cores).

    A: [N, C (lmax+1)^2] float32 CUDA tensor (node-row layout, C in 32, 64, 96, 128);
    Ws: [nu - 1, node_ladder_full_step_floats(lmax, C)] (nu - 1 may be 0). Returns out like A.
    """
    torch = _torch()
    _need_cuda(A, Ws)
    A, Ws = _f32(A), _f32(Ws)
    n, dim = A.shape
    c = dim // ((lmax + 1) ** 2)
    nu = Ws.shape[0] + 1
    lib = load_library()
    if out is None:
        out = torch.empty_like(A)
    need = int(lib.etp_node_ladder_full_workspace_bytes(int(lmax), c, n))
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=A.device)
    _check(lib.etp_node_ladder_full(int(lmax), c, n, nu, _ptr(A), _ptr(Ws) if nu > 1 else None, _ptr(out),
                                    _ptr(workspace), workspace.numel(), _stream(A.device)), "etp_node_ladder_full")
    return out


def edge_conv_function():
    """torch.autograd.Function: out = conv(x, edge_vec, W); gradients for x, edge_vec and W."""
    torch = _torch()

    class _EdgeConvFn(torch.autograd.Function):
        @staticmethod
        def forward(ctx, conv, graph, x, edge_vec, W):
            g = Graph(graph.n_nodes, graph.n_edges, graph.row_ptr, graph.sender, edge_vec.detach(),
                      graph.t_row_ptr, graph.t_perm)
            ctx.conv, ctx.graph = conv, g
            ctx.save_for_backward(x, W)
            return conv.forward(g, x.detach(), W.detach())

        @staticmethod
        def backward(ctx, grad_out):
            x, W = ctx.saved_tensors
            go = grad_out.contiguous()
            gx = gv = gW = None
            if ctx.needs_input_grad[2] or ctx.needs_input_grad[3]:
                gx, gv = ctx.conv.backward(ctx.graph, x.detach(), W.detach(), go, ctx.needs_input_grad[2],
                                           ctx.needs_input_grad[3])
            if ctx.needs_input_grad[4]:
                gW = ctx.conv.backward_weights(ctx.graph, x.detach(), go).reshape(W.shape)
            return None, None, gx, gv, gW

    return _EdgeConvFn
