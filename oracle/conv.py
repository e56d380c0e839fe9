"""Edge tensor-product convolution: forward and analytic VJP (oracle; test infrastructure only).

The operation, as the workload description states it and in the notation of
the pages (Fig. 3 caption of "FlashCart": path-reduced products summed inside
the kernel with one scalar weight per path and feature channel; Fig. D1: node
rows hold rank blocks at offsets off(l), channels contiguous):

    for each receiver i, for each edge e = (i <- j, S) of row i:
        r = edge vector (receiver -> sender), d = |r|, n = r / d
        Y_l2 = real SH of n (component normalisation), l2 = 0..sh_lmax
        R_b  = B_b(d) u(d / r_c),  b = 1..n_basis
        for each path p = (l1 block of irreps_in, l2, l3 block of irreps_out), channel u:
            w_{e,p,u} = sum_b R_b W[b, p, u]
            out[i, l3, m3, u] += w_{e,p,u} sum_{m1,m2} C^{l1 l2 l3}_{m1 m2 m3} x[j, l1, m1, u] Y_{l2 m2}(n)

"uvu": the output channel equals the input channel; the harmonics have
multiplicity one. Paths are all (block_in, l2, block_out) with the triangle
rule, parity p1 (-1)^l2 = p3 and equal multiplicities of the two blocks (the
channel pairing needs them), in lexicographic (block_in, l2, block_out) order
("Fast and Accurate Foundation Models...", section VII: irreps parity
restricted to that of the harmonics is the fast case; NequIP-style per-l
channel counts of "High-performance training and inference...", Table 1, and
paths with l1 + l2 + l3 odd are the general one). W has layout
[n_basis, weight_numel]: path p owns the mul_p columns starting at
woff_p = sum of the earlier paths' multiplicities ([n_basis, n_paths, C] when
every block has C channels). Node rows: blocks in irreps order, each block
[m][u] (m = -l..l, u contiguous).

Vectorised with numpy over edges, one path at a time; the receiver sum is a
plain scatter-add (np.add.at). No blocking, fusion or reordering beyond that.
"""
import re
from dataclasses import dataclass, field

import numpy as np

from .cg import cg_real
from .radial import radial, radial_deriv
from .sh import sh_real, sh_real_grad


def parse_irreps(s):
    """'64x0e+64x1o' -> [(64, 0, +1), (64, 1, -1)]. A bare '1o' means multiplicity 1."""
    blocks = []
    for term in s.replace(" ", "").split("+"):
        m = re.fullmatch(r"(?:(\d+)x)?(\d+)([eo])", term)
        if not m:
            raise ValueError(f"bad irreps term {term!r}")
        mul = int(m.group(1)) if m.group(1) else 1
        blocks.append((mul, int(m.group(2)), 1 if m.group(3) == "e" else -1))
    return blocks


@dataclass
class ConvSpec:
    irreps_in: str
    sh_lmax: int
    irreps_out: str
    n_basis: int
    r_cut: float
    blocks_in: list = field(init=False)
    blocks_out: list = field(init=False)
    paths: list = field(init=False)
    channels: int = field(init=False)      # the common multiplicity, or None when blocks differ
    path_mul: list = field(init=False)
    woff: list = field(init=False)
    weight_numel: int = field(init=False)  # columns of W (per basis function)

    def __post_init__(self):
        self.blocks_in = parse_irreps(self.irreps_in)
        self.blocks_out = parse_irreps(self.irreps_out)
        muls = {b[0] for b in self.blocks_in + self.blocks_out}
        self.channels = muls.pop() if len(muls) == 1 else None
        self.paths = []
        for bi, (m1, l1, p1) in enumerate(self.blocks_in):
            for l2 in range(self.sh_lmax + 1):
                for bo, (m3, l3, p3) in enumerate(self.blocks_out):
                    if abs(l1 - l2) <= l3 <= l1 + l2 and p1 * (-1) ** l2 == p3 and m1 == m3:
                        self.paths.append((bi, l2, bo))
        self.path_mul = [self.blocks_in[bi][0] for bi, _, _ in self.paths]
        self.woff = [int(v) for v in np.cumsum([0] + self.path_mul)[:-1]]
        self.weight_numel = int(sum(self.path_mul))

    @staticmethod
    def _offsets(blocks):
        off, o = [], 0
        for mul, l, _ in blocks:
            off.append(o)
            o += mul * (2 * l + 1)
        return off, o

    @property
    def dim_in(self):
        return self._offsets(self.blocks_in)[1]

    @property
    def dim_out(self):
        return self._offsets(self.blocks_out)[1]

    def in_slice(self, b):
        off = self._offsets(self.blocks_in)[0][b]
        return slice(off, off + self.blocks_in[b][0] * (2 * self.blocks_in[b][1] + 1))

    def out_slice(self, b):
        off = self._offsets(self.blocks_out)[0][b]
        return slice(off, off + self.blocks_out[b][0] * (2 * self.blocks_out[b][1] + 1))

    def w_slice(self, p):
        """Columns of W (and of the per-edge weights w) that belong to path p."""
        return slice(self.woff[p], self.woff[p] + self.path_mul[p])

    def path_ls(self, p):
        bi, l2, bo = self.paths[p]
        return self.blocks_in[bi][1], l2, self.blocks_out[bo][1]


def _edge_geometry(spec, edge_vec):
    vec = np.asarray(edge_vec)
    if vec.dtype == np.float32:
        vec = vec.astype(np.float64)
    d = np.sqrt(vec[:, 0] * vec[:, 0] + vec[:, 1] * vec[:, 1] + vec[:, 2] * vec[:, 2])
    ys = [sh_real(l, vec) for l in range(spec.sh_lmax + 1)]
    rad = radial(d, spec.n_basis, np.float64(np.float32(spec.r_cut)))
    return vec, d, ys, rad


def _edge_rows(row_ptr, receivers):
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    n = len(row_ptr) - 1
    if receivers is None:
        receivers = np.arange(n)
    receivers = np.asarray(receivers, dtype=np.int64)
    counts = row_ptr[receivers + 1] - row_ptr[receivers]
    edges = np.concatenate([np.arange(row_ptr[i], row_ptr[i + 1]) for i in receivers]) \
        if len(receivers) else np.zeros(0, dtype=np.int64)
    local = np.repeat(np.arange(len(receivers)), counts)
    return receivers, edges.astype(np.int64), local


def _mask_bits(path_mask, n_p):
    """[E, n_p] 0/1 array from per-edge masks (bit p of path_mask[e] set: path p is on)."""
    m = np.asarray(path_mask, dtype=np.uint64)
    return ((m[:, None] >> np.arange(n_p, dtype=np.uint64)[None, :]) & np.uint64(1)).astype(np.float64)


def conv_forward(spec, row_ptr, sender, edge_vec, x, W, receivers=None, path_mask=None):
    """out[i] for i in ``receivers`` (default: all). Returns [len(receivers), dim_out].

    x: [N, dim_in]; W: [n_basis, weight_numel] (or [n_basis, n_paths, C]). Inputs are upcast to float64
    (complex inputs stay complex, for complex-step checks).
    path_mask: optional per-edge integers (canonical order); path p contributes for edge e only
    when bit p of path_mask[e] is set (per-edge path selection, as in adaptive-depth models).
    """
    receivers, edges, local = _edge_rows(row_ptr, receivers)
    sender = np.asarray(sender, dtype=np.int64)[edges]
    xs_all = np.asarray(x)
    xs_all = xs_all.astype(np.float64) if xs_all.dtype == np.float32 else xs_all
    W = np.asarray(W, dtype=np.float64)
    vec, d, ys, rad = _edge_geometry(spec, np.asarray(edge_vec)[edges])
    n_e, n_p = len(edges), len(spec.paths)
    w = rad @ W.reshape(spec.n_basis, spec.weight_numel)          # [E, weight_numel]
    mbits = _mask_bits(np.asarray(path_mask)[edges], n_p) if path_mask is not None else None
    dtype = np.result_type(vec, xs_all, np.float64)
    out = np.zeros((len(receivers), spec.dim_out), dtype=dtype)
    for p, (bi, l2, bo) in enumerate(spec.paths):
        l1, _, l3 = spec.path_ls(p)
        c = spec.path_mul[p]
        cg = cg_real(l1, l2, l3)
        wp = w[:, spec.w_slice(p)]
        if mbits is not None:
            wp = wp * mbits[:, p, None]
        xj = xs_all[sender][:, spec.in_slice(bi)].reshape(n_e, 2 * l1 + 1, c)
        msg = np.einsum("abc,eb,eau->ecu", cg, ys[l2], xj) * wp[:, None, :]
        blk = np.zeros((len(receivers), 2 * l3 + 1, c), dtype=dtype)
        np.add.at(blk, local, msg)
        out[:, spec.out_slice(bo)] += blk.reshape(len(receivers), -1)
    return out


def conv_vjp(spec, row_ptr, sender, edge_vec, x, W, grad_out, path_mask=None):
    """Exact VJP of ``conv_forward`` (all receivers) with respect to x and the edge vectors.

    Returns grad_x [N, dim_in] and grad_edge_vec [E, 3] (float64).

    With s_{e,p,u}[m3] = sum C x Y and L = <grad_out, out>:
      dL/dx[j, l1, m1, u]   = sum_{e: send=j} sum_p w sum_{m2,m3} C Y g[recv, l3, m3, u]
      dL/dw_{e,p,u}          = sum_m3 g[recv, l3, m3, u] s_{e,p,u}[m3]
      dL/dY_{l2,m2}(e)       = sum_{p,u} w sum_{m1,m3} C x[send, l1, m1, u] g[recv, l3, m3, u]
      dL/dR_b(e)             = sum_{p,u} W[b,p,u] dL/dw_{e,p,u}
      dL/dr_e                = (sum_b dL/dR_b dR_b/dd) r/d + sum_{l2,m2} dL/dY dY/dr
    """
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    n_nodes = len(row_ptr) - 1
    sender = np.asarray(sender, dtype=np.int64)
    n_e = len(sender)
    receiver = np.repeat(np.arange(n_nodes), np.diff(row_ptr))
    x = np.asarray(x, dtype=np.float64)
    g = np.asarray(grad_out, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    vec, d, ys, rad = _edge_geometry(spec, edge_vec)
    n_p = len(spec.paths)
    Wf = W.reshape(spec.n_basis, spec.weight_numel)
    w = rad @ Wf                                                   # [E, weight_numel]
    mbits = _mask_bits(path_mask, n_p) if path_mask is not None else np.ones((n_e, n_p))
    grad_x = np.zeros((n_nodes, spec.dim_in))
    grad_w = np.zeros((n_e, spec.weight_numel))
    grad_y = [np.zeros((n_e, 2 * l + 1)) for l in range(spec.sh_lmax + 1)]
    for p, (bi, l2, bo) in enumerate(spec.paths):
        l1, _, l3 = spec.path_ls(p)
        c = spec.path_mul[p]
        cg = cg_real(l1, l2, l3)
        wp = w[:, spec.w_slice(p)] * mbits[:, p, None]
        xj = x[sender][:, spec.in_slice(bi)].reshape(n_e, 2 * l1 + 1, c)
        gi = g[receiver][:, spec.out_slice(bo)].reshape(n_e, 2 * l3 + 1, c)
        gw = gi * wp[:, None, :]
        gx_e = np.einsum("abc,eb,ecu->eau", cg, ys[l2], gw)
        blk = np.zeros((n_nodes, 2 * l1 + 1, c))
        np.add.at(blk, sender, gx_e)
        grad_x[:, spec.in_slice(bi)] += blk.reshape(n_nodes, -1)
        s = np.einsum("abc,eb,eau->ecu", cg, ys[l2], xj)
        # a masked path's weight does not reach the output
        grad_w[:, spec.w_slice(p)] = (gi * s).sum(axis=1) * mbits[:, p, None]
        grad_y[l2] += np.einsum("abc,eau,ecu->eb", cg, xj, gw)
    grad_r = grad_w @ Wf.T
    grad_d = (grad_r * radial_deriv(d, spec.n_basis, np.float64(np.float32(spec.r_cut)))).sum(axis=1)
    grad_vec = grad_d[:, None] * vec / d[:, None]
    for l in range(spec.sh_lmax + 1):
        grad_vec += np.einsum("em,emk->ek", grad_y[l], sh_real_grad(l, vec))
    return grad_x, grad_vec


def conv_vjp_weights(spec, row_ptr, sender, edge_vec, x, grad_out):
    """Exact gradient of L = <grad_out, conv_forward(...)> with respect to W (float64).

    The forward is linear in W through w_{e,p,u} = sum_b R_b(d_e) W[b,p,u], so
      dL/dW[b,p,u] = sum_e R_b(d_e) dL/dw_{e,p,u},
      dL/dw_{e,p,u} = sum_m3 g[recv, l3, m3, u] sum_{m1,m2} C[m1,m2,m3] x[send, l1, m1, u] Y_{l2 m2}(e).
    Returns [n_basis, n_paths, C] when every block has C channels, else [n_basis, weight_numel].
    """
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    n_nodes = len(row_ptr) - 1
    sender = np.asarray(sender, dtype=np.int64)
    n_e = len(sender)
    receiver = np.repeat(np.arange(n_nodes), np.diff(row_ptr))
    x = np.asarray(x, dtype=np.float64)
    g = np.asarray(grad_out, dtype=np.float64)
    _, _, ys, rad = _edge_geometry(spec, edge_vec)
    n_p = len(spec.paths)
    dw_edge = np.zeros((n_e, spec.weight_numel))
    for p, (bi, l2, bo) in enumerate(spec.paths):
        l1, _, l3 = spec.path_ls(p)
        c = spec.path_mul[p]
        cg = cg_real(l1, l2, l3)
        xj = x[sender][:, spec.in_slice(bi)].reshape(n_e, 2 * l1 + 1, c)
        gi = g[receiver][:, spec.out_slice(bo)].reshape(n_e, 2 * l3 + 1, c)
        s = np.einsum("abc,eb,eau->ecu", cg, ys[l2], xj)
        dw_edge[:, spec.w_slice(p)] = (gi * s).sum(axis=1)
    dw = rad.T @ dw_edge
    return dw.reshape(spec.n_basis, n_p, spec.channels) if spec.channels is not None else dw


def flop_counts(spec):
    """Algorithmic operation counts per edge of the plain definition (FMA = 2 flops).

    fwd_tp     : sum_p 2 (nnz_p + 2 l3 + 1) mul_p    -- CG contraction with c_k = C_k Y, then w * s
    radial_proj: 2 n_basis weight_numel              -- w = R W
    bwd_tp     : sum_p 2 (3 nnz_p + 2 (2 l3 + 1)) mul_p -- grad_x, grad_w and grad_Y contractions
    (with one multiplicity C for every block: 2 (nnz + sum_p(2 l3 + 1)) C and so on).
    Also returns nnz (real-CG nonzeros over the path set) and sum_2l3p1.
    """
    nnz = s3 = fwd = bwd = 0
    for p in range(len(spec.paths)):
        l1, l2, l3 = spec.path_ls(p)
        nz = int(np.count_nonzero(cg_real(l1, l2, l3)))
        nnz += nz
        s3 += 2 * l3 + 1
        fwd += 2 * (nz + 2 * l3 + 1) * spec.path_mul[p]
        bwd += 2 * (3 * nz + 2 * (2 * l3 + 1)) * spec.path_mul[p]
    return {
        "nnz": nnz,
        "sum_2l3p1": s3,
        "fwd_tp": fwd,
        "radial_proj": 2 * spec.n_basis * spec.weight_numel,
        "bwd_tp": bwd,
    }
