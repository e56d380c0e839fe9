"""Build-time generator of the unrolled per-path device code (``generated/etp_paths.h``).

Emits, for every supported l_max (in = SH = out = L):
  * the real spherical harmonics Y_lm(n) of a unit vector as explicit polynomials
    (component normalisation, sum_m Y_lm^2 = 2l + 1, m = -l..l, z polar), and the
    contraction sum_m gY_m dY_m/dr needed by the backward pass;
  * the path list (l1, l2, l3), lexicographic, triangle rule, l1 + l2 + l3 even;
  * per path, the real-basis Clebsch-Gordan nonzeros as float immediates inside
    straight-line forward and backward contraction code, and the per-path factor
    of the weight gradient, sum_{m1,m3} x[l1 m1] (sum_m2 C Y[l2 m2]) g[l3 m3];
  * the node-local path-reduced product of two feature rows (tp_node_L);
  * for general irreps (any multiplicities and parities, rank <= 4), one forward and one
    backward contraction per coupling (l1, l2, l3), even and odd l1 + l2 + l3, over one
    channel with the block stride as an argument, dispatched by a coupling index; and the
    harmonics up to l = 4.

Independent of the float64 oracle by construction: Clebsch-Gordan values come
from ``sympy.physics.wigner.clebsch_gordan`` and the harmonic polynomials from a
least-squares fit of homogeneous polynomials to ``scipy.special.sph_harm_y``
(a homogeneous polynomial of degree l is fixed by its values on the sphere),
each moved to the real basis by the change of basis written out below.

Run:  python gen_paths.py  (writes generated/etp_paths.h next to this file)
"""
import itertools
import math
import os
import struct
import sys

import numpy as np
import scipy.special as sps
from sympy import N as sym_n
from sympy.physics.wigner import clebsch_gordan

LMAX_SUPPORTED = (1, 2, 3)
HERE = os.path.dirname(os.path.abspath(__file__))


# ---------------------------------------------------------------- bases

def complex_to_real(l):
    """U with Y_real = U Y_complex; real m>0 ~ cos(m phi), m<0 ~ sin(|m| phi)."""
    u = np.zeros((2 * l + 1, 2 * l + 1), dtype=complex)
    r = math.sqrt(0.5)
    u[l, l] = 1.0
    for m in range(1, l + 1):
        sgn = -1.0 if m % 2 else 1.0
        u[l + m, l + m] = sgn * r
        u[l + m, l - m] = r
        u[l - m, l - m] = 1j * r
        u[l - m, l + m] = -1j * sgn * r
    return u


def real_cg(l1, l2, l3):
    c = np.zeros((2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1), dtype=complex)
    for m1 in range(-l1, l1 + 1):
        for m2 in range(-l2, l2 + 1):
            m3 = m1 + m2
            if abs(m3) <= l3:
                c[m1 + l1, m2 + l2, m3 + l3] = float(sym_n(clebsch_gordan(l1, l2, l3, m1, m2, m3), 30))
    u1, u2, u3 = complex_to_real(l1), complex_to_real(l2), complex_to_real(l3)
    r = np.einsum("ai,bj,ck,ijk->abc", u1.conj(), u2.conj(), u3, c)
    assert np.abs(r.imag).max() < 1e-12
    r = r.real
    r[np.abs(r) < 1e-12] = 0.0
    return r


def real_cg_any(l1, l2, l3):
    """Real coupling for any triangle triple: the real tensor for l1 + l2 + l3 even; for odd sums
    the change of basis gives i times a real tensor, and that real tensor is the coupling."""
    c = np.zeros((2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1), dtype=complex)
    for m1 in range(-l1, l1 + 1):
        for m2 in range(-l2, l2 + 1):
            m3 = m1 + m2
            if abs(m3) <= l3:
                c[m1 + l1, m2 + l2, m3 + l3] = float(sym_n(clebsch_gordan(l1, l2, l3, m1, m2, m3), 30))
    u1, u2, u3 = complex_to_real(l1), complex_to_real(l2), complex_to_real(l3)
    r = np.einsum("ai,bj,ck,ijk->abc", u1.conj(), u2.conj(), u3, c)
    if (l1 + l2 + l3) % 2 == 0:
        assert np.abs(r.imag).max() < 1e-12
        r = r.real
    else:
        assert np.abs(r.real).max() < 1e-12
        r = r.imag
    r = r.copy()
    r[np.abs(r) < 1e-12] = 0.0
    return r


def monomials(l):
    return [(a, b, l - a - b) for a in range(l, -1, -1) for b in range(l - a, -1, -1)]


def sh_polynomials(l):
    """Coefficients over ``monomials(l)`` of Y_lm (component normalised), rows m=-l..l."""
    rng = np.random.default_rng(1234 + l)
    v = rng.standard_normal((400, 3))
    v /= np.linalg.norm(v, axis=1, keepdims=True)
    theta, phi = np.arccos(np.clip(v[:, 2], -1, 1)), np.arctan2(v[:, 1], v[:, 0])
    yc = np.stack([sps.sph_harm_y(l, m, theta, phi) for m in range(-l, l + 1)], axis=0)
    yr = (complex_to_real(l) @ yc).real * math.sqrt(4.0 * math.pi)
    mons = monomials(l)
    a = np.stack([v[:, 0] ** p * v[:, 1] ** q * v[:, 2] ** s for p, q, s in mons], axis=1)
    coef, *_ = np.linalg.lstsq(a, yr.T, rcond=None)
    assert np.abs(a @ coef - yr.T).max() < 1e-12, l
    coef[np.abs(coef) < 1e-12] = 0.0
    return coef.T  # [2l+1, n_monomials]


# ---------------------------------------------------------------- emit helpers

def repr_f32(f):
    # hexadecimal float literal, exact for float32 values
    return float.hex(float(f)) + "f"


def idx(l, m):
    return l * l + l + m


def paths_for(lmax):
    return [(l1, l2, l3) for l1 in range(lmax + 1) for l2 in range(lmax + 1) for l3 in range(lmax + 1)
            if abs(l1 - l2) <= l3 <= l1 + l2 and (l1 + l2 + l3) % 2 == 0]


def mono_expr(p, q, s, names=("nx", "ny", "nz")):
    parts = []
    for n, e in zip(names, (p, q, s)):
        parts += [n] * e
    return "*".join(parts) if parts else "1.0f"


# ---------------------------------------------------------------- SH code

def emit_sh(out, lmax):
    out.append(f"// real spherical harmonics up to l = {lmax}: Y[l*l + l + m] of the unit vector (nx, ny, nz)")
    out.append(f"__device__ __forceinline__ void sh_eval_{lmax}(float nx, float ny, float nz, float* Y) {{")
    out.append("  Y[0] = 1.0f;")
    for l in range(1, lmax + 1):
        coef = sh_polynomials(l)
        mons = monomials(l)
        for m in range(-l, l + 1):
            terms = [(coef[m + l, k], mons[k]) for k in range(len(mons)) if coef[m + l, k] != 0.0]
            expr = " + ".join(f"{repr_f32(np.float32(c))}*({mono_expr(*mo)})" for c, mo in terms)
            out.append(f"  Y[{idx(l, m)}] = {expr};")
    out.append("}")
    # gradient contraction: given gY (dL/dY), returns G = sum_m gY_m grad P_m(n) and
    # S = sum_m gY_m l P_m(n); then dL/dr = (G - S n) / d
    out.append(f"__device__ __forceinline__ void sh_grad_{lmax}(float nx, float ny, float nz, const float* gY,")
    out.append("                                              float& Gx, float& Gy, float& Gz, float& S) {")
    out.append("  Gx = 0.0f; Gy = 0.0f; Gz = 0.0f; S = 0.0f;")
    for l in range(1, lmax + 1):
        coef = sh_polynomials(l)
        mons = monomials(l)
        for m in range(-l, l + 1):
            i = idx(l, m)
            terms = [(coef[m + l, k], mons[k]) for k in range(len(mons)) if coef[m + l, k] != 0.0]
            gx, gy, gz, pv = [], [], [], []
            for c, (p, q, s) in terms:
                pv.append(f"{repr_f32(np.float32(c))}*({mono_expr(p, q, s)})")
                if p:
                    gx.append(f"{repr_f32(np.float32(c * p))}*({mono_expr(p - 1, q, s)})")
                if q:
                    gy.append(f"{repr_f32(np.float32(c * q))}*({mono_expr(p, q - 1, s)})")
                if s:
                    gz.append(f"{repr_f32(np.float32(c * s))}*({mono_expr(p, q, s - 1)})")
            out.append(f"  {{ const float g = gY[{i}];")
            for name, lst in (("Gx", gx), ("Gy", gy), ("Gz", gz)):
                if lst:
                    out.append(f"    {name} = fmaf(g, {' + '.join(lst)}, {name});")
            out.append(f"    S = fmaf(g * {float(l):.1f}f, {' + '.join(pv)}, S); }}")
    out.append("}")


# ---------------------------------------------------------------- path code

def emit_paths(out, lmax):
    paths = paths_for(lmax)
    P = len(paths)
    D = (lmax + 1) ** 2
    cgs = [real_cg(*p) for p in paths]
    nnz = sum(int(np.count_nonzero(c)) for c in cgs)
    s3 = sum(2 * l3 + 1 for _, _, l3 in paths)
    out.append(f"// ---- l_max = {lmax}: {P} paths, {nnz} real-CG nonzeros")
    out.append(f"template <> struct PathSet<{lmax}> {{")
    out.append(f"  static constexpr int L = {lmax};")
    out.append(f"  static constexpr int P = {P};")
    out.append(f"  static constexpr int D = {D};")
    out.append(f"  static constexpr int NNZ = {nnz};")
    out.append(f"  static constexpr int SUM_2L3P1 = {s3};")
    out.append("};")
    trip = ", ".join(f"{a},{b},{c}" for a, b, c in paths)
    out.append(f"static const int kPathL_{lmax}[{3 * P}] = {{{trip}}};")

    # forward: acc[l3 m3][k] += w_p[k] * sum_{m1,m2} C Y[l2 m2] x[l1 m1][k]
    out.append("template <int K, class WF>")
    out.append(f"__device__ __forceinline__ void tp_fwd_{lmax}(const float* Y, WF&& wfetch,")
    out.append(f"    const float (&x)[{D}][K], float (&acc)[{D}][K]) {{")
    for p, ((l1, l2, l3), c) in enumerate(zip(paths, cgs)):
        out.append(f"  {{ // path {p}: ({l1},{l2},{l3})")
        out.append(f"    float wp[K];")
        out.append(f"    if (fetch(wfetch, IC<{p}>{{}}, wp)) {{")
        # M[m3][m1] = sum_m2 C[m1,m2,m3] Y[l2,m2]
        mnz = []
        for m3 in range(2 * l3 + 1):
            for m1 in range(2 * l1 + 1):
                terms = [(c[m1, m2, m3], idx(l2, m2 - l2)) for m2 in range(2 * l2 + 1) if c[m1, m2, m3] != 0.0]
                if not terms:
                    continue
                if l2 == 0:
                    e = repr_f32(np.float32(terms[0][0]))
                else:
                    e = " + ".join(f"{repr_f32(np.float32(v))}*Y[{i}]" for v, i in terms)
                out.append(f"    const float M{m3}_{m1} = {e};")
                mnz.append((m3, m1))
        scale_x = (2 * l1 + 1) < (2 * l3 + 1)
        out.append("    #pragma unroll")
        out.append("    for (int k = 0; k < K; ++k) {")
        if scale_x:
            for m1 in range(2 * l1 + 1):
                out.append(f"      const float xs{m1} = wp[k] * x[{idx(l1, m1 - l1)}][k];")
            for m3 in range(2 * l3 + 1):
                for (a, b) in mnz:
                    if a == m3:
                        out.append(f"      acc[{idx(l3, m3 - l3)}][k] = fmaf(M{a}_{b}, xs{b}, acc[{idx(l3, m3 - l3)}][k]);")
        else:
            for m3 in range(2 * l3 + 1):
                row = [(a, b) for (a, b) in mnz if a == m3]
                if not row:
                    continue
                a, b = row[0]
                out.append(f"      float s{m3} = M{a}_{b} * x[{idx(l1, b - l1)}][k];")
                for a, b in row[1:]:
                    out.append(f"      s{m3} = fmaf(M{a}_{b}, x[{idx(l1, b - l1)}][k], s{m3});")
                out.append(f"      acc[{idx(l3, m3 - l3)}][k] = fmaf(wp[k], s{m3}, acc[{idx(l3, m3 - l3)}][k]);")
        out.append("    }")
        out.append("    }")
        out.append("  }")
    out.append("}")

    # backward (one edge, K channels):
    #   v[m1]   = sum_m3 M[m3][m1] g[l3 m3]
    #   gx      += w v;   gw = sum_m1 x[l1 m1] v[m1];   accd += wd gw
    #   gY[l2 m2] += w sum_{m1,m3} C[m1,m2,m3] x[l1 m1] g[l3 m3]
    out.append("template <int K, class WF>")
    out.append(f"__device__ __forceinline__ void tp_bwd_{lmax}(const float* Y, WF&& wfetch,")
    out.append(f"    const float (&x)[{D}][K], const float (&g)[{D}][K], float (&gx)[{D}][K],")
    out.append(f"    float* gY, float& accd) {{")
    for p, ((l1, l2, l3), c) in enumerate(zip(paths, cgs)):
        out.append(f"  {{ // path {p}: ({l1},{l2},{l3})")
        out.append(f"    float wp[K], wdp[K];")
        out.append(f"    if (fetch(wfetch, IC<{p}>{{}}, wp, wdp)) {{")
        mnz = []
        for m3 in range(2 * l3 + 1):
            for m1 in range(2 * l1 + 1):
                terms = [(c[m1, m2, m3], idx(l2, m2 - l2)) for m2 in range(2 * l2 + 1) if c[m1, m2, m3] != 0.0]
                if not terms:
                    continue
                if l2 == 0:
                    e = repr_f32(np.float32(terms[0][0]))
                else:
                    e = " + ".join(f"{repr_f32(np.float32(v))}*Y[{i}]" for v, i in terms)
                out.append(f"    const float M{m3}_{m1} = {e};")
                mnz.append((m3, m1))
        out.append("    #pragma unroll")
        out.append("    for (int k = 0; k < K; ++k) {")
        for m1 in range(2 * l1 + 1):
            col = [(a, b) for (a, b) in mnz if b == m1]
            if not col:
                out.append(f"      const float v{m1} = 0.0f;")
                continue
            a, b = col[0]
            out.append(f"      float v{m1} = M{a}_{b} * g[{idx(l3, a - l3)}][k];")
            for a, b in col[1:]:
                out.append(f"      v{m1} = fmaf(M{a}_{b}, g[{idx(l3, a - l3)}][k], v{m1});")
        for m1 in range(2 * l1 + 1):
            out.append(f"      gx[{idx(l1, m1 - l1)}][k] = fmaf(wp[k], v{m1}, gx[{idx(l1, m1 - l1)}][k]);")
        out.append(f"      float gw = x[{idx(l1, -l1)}][k] * v0;")
        for m1 in range(1, 2 * l1 + 1):
            out.append(f"      gw = fmaf(x[{idx(l1, m1 - l1)}][k], v{m1}, gw);")
        out.append("      accd = fmaf(wdp[k], gw, accd);")
        if l2 > 0:
            # gY[l2 m2] += w * sum C x g
            for m2 in range(2 * l2 + 1):
                terms = [(c[m1, m2, m3], m1, m3) for m1 in range(2 * l1 + 1) for m3 in range(2 * l3 + 1)
                         if c[m1, m2, m3] != 0.0]
                if not terms:
                    continue
                v, a, b = terms[0]
                out.append(f"      float q{m2} = {repr_f32(np.float32(v))} * (x[{idx(l1, a - l1)}][k] * g[{idx(l3, b - l3)}][k]);")
                for v, a, b in terms[1:]:
                    out.append(f"      q{m2} = fmaf({repr_f32(np.float32(v))}, x[{idx(l1, a - l1)}][k] * g[{idx(l3, b - l3)}][k], q{m2});")
                out.append(f"      gY[{idx(l2, m2 - l2)}] = fmaf(wp[k], q{m2}, gY[{idx(l2, m2 - l2)}]);")
        out.append("    }")
        out.append("    }")
        out.append("  }")
    out.append("}")

    # weight gradient factor (one edge, K channels): gw_p[k] = sum_{m1,m3} x[l1 m1] M[m3][m1] g[l3 m3],
    # evaluated as x . (M^T g) or g . (M x), whichever side is shorter; handed to gsink per path.
    out.append("template <int K, class GS>")
    out.append(f"__device__ __forceinline__ void tp_gw_{lmax}(const float* Y, const float (&x)[{D}][K],")
    out.append(f"    const float (&g)[{D}][K], GS&& gsink) {{")
    for p, ((l1, l2, l3), c) in enumerate(zip(paths, cgs)):
        out.append(f"  {{ // path {p}: ({l1},{l2},{l3})")
        mnz = []
        for m3 in range(2 * l3 + 1):
            for m1 in range(2 * l1 + 1):
                terms = [(c[m1, m2, m3], idx(l2, m2 - l2)) for m2 in range(2 * l2 + 1) if c[m1, m2, m3] != 0.0]
                if not terms:
                    continue
                if l2 == 0:
                    e = repr_f32(np.float32(terms[0][0]))
                else:
                    e = " + ".join(f"{repr_f32(np.float32(v))}*Y[{i}]" for v, i in terms)
                out.append(f"    const float M{m3}_{m1} = {e};")
                mnz.append((m3, m1))
        out.append("    float gw[K];")
        out.append("    #pragma unroll")
        out.append("    for (int k = 0; k < K; ++k) {")
        via_v = (2 * l1 + 1) <= (2 * l3 + 1)
        first = True
        if via_v:
            for m1 in range(2 * l1 + 1):
                col = [(a, b) for (a, b) in mnz if b == m1]
                if not col:
                    continue
                a, b = col[0]
                out.append(f"      float v{m1} = M{a}_{b} * g[{idx(l3, a - l3)}][k];")
                for a, b in col[1:]:
                    out.append(f"      v{m1} = fmaf(M{a}_{b}, g[{idx(l3, a - l3)}][k], v{m1});")
                if first:
                    out.append(f"      float t = x[{idx(l1, m1 - l1)}][k] * v{m1};")
                    first = False
                else:
                    out.append(f"      t = fmaf(x[{idx(l1, m1 - l1)}][k], v{m1}, t);")
        else:
            for m3 in range(2 * l3 + 1):
                row = [(a, b) for (a, b) in mnz if a == m3]
                if not row:
                    continue
                a, b = row[0]
                out.append(f"      float s{m3} = M{a}_{b} * x[{idx(l1, b - l1)}][k];")
                for a, b in row[1:]:
                    out.append(f"      s{m3} = fmaf(M{a}_{b}, x[{idx(l1, b - l1)}][k], s{m3});")
                if first:
                    out.append(f"      float t = g[{idx(l3, m3 - l3)}][k] * s{m3};")
                    first = False
                else:
                    out.append(f"      t = fmaf(g[{idx(l3, m3 - l3)}][k], s{m3}, t);")
        out.append("      gw[k] = t;" if not first else "      gw[k] = 0.0f;")
        out.append("    }")
        out.append(f"    gsink(IC<{p}>{{}}, gw);")
        out.append("  }")
    out.append("}")
    return P, nnz, s3


# ---------------------------------------------------------------- node-local product
def emit_node(out, lmax):
    """acc[l3 m3][k] += w_p[k] sum_{m1,m2} C[m1,m2,m3] b[l1 m1][k] a[l2 m2][k] for every path: the
    path-reduced product of two node features, one channel per k (FlashCart Fig. 3b)."""
    paths = paths_for(lmax)
    D = (lmax + 1) ** 2
    ent = path_m_entries(lmax)
    out.append("template <int K, class WF>")
    out.append(f"__device__ __forceinline__ void tp_node_{lmax}(const float (&b)[{D}][K], const float (&a)[{D}][K],")
    out.append(f"    WF&& wfetch, float (&acc)[{D}][K]) {{")
    for p, (l1, l2, l3) in enumerate(paths):
        out.append(f"  {{ // path {p}: ({l1},{l2},{l3})")
        out.append("    float wp[K];")
        out.append(f"    wfetch(IC<{p}>{{}}, wp);")
        out.append("    #pragma unroll")
        out.append("    for (int k = 0; k < K; ++k) {")
        for m3 in range(2 * l3 + 1):
            row = [(m1, terms) for (a3, m1, terms) in ent[p] if a3 == m3]
            if not row:
                continue
            first = True
            for m1, terms in row:
                mexpr = " + ".join(f"{repr_f32(np.float32(v))}*a[{i}][k]" for v, i in terms)
                if first:
                    out.append(f"      float s{m3} = ({mexpr}) * b[{idx(l1, m1 - l1)}][k];")
                    first = False
                else:
                    out.append(f"      s{m3} = fmaf({mexpr}, b[{idx(l1, m1 - l1)}][k], s{m3});")
            out.append(f"      acc[{idx(l3, m3 - l3)}][k] = fmaf(wp[k], s{m3}, acc[{idx(l3, m3 - l3)}][k]);")
        out.append("    }")
        out.append("  }")
    out.append("}")


# ---------------------------------------------------------------- full product ladder
def emit_ladder_t(out, lmax):
    """The unweighted per-path products of the full ladder for one channel (FlashCart Fig. E1 (b)):
    t[kLadderOff[l3] + m3 * kLadderP[l3] + j] = sum_{m1,m2} C[m1,m2,m3] b[l1 m1] a[l2 m2], j = the
    path's index among the paths of output rank l3 (path order). Each (l3, m3) row of j values is
    the K dimension of that output component's mixing matrix."""
    paths = paths_for(lmax)
    D = (lmax + 1) ** 2
    ent = path_m_entries(lmax)
    by_rank = [[p for p, (_, _, c) in enumerate(paths) if c == l3] for l3 in range(lmax + 1)]
    offs, nt = [], 0
    for l3 in range(lmax + 1):
        offs.append(nt)
        nt += (2 * l3 + 1) * len(by_rank[l3])
    out.append(f"template <> struct LadderShape<{lmax}> {{")
    out.append(f"  static constexpr int NT = {nt};   // products per node and channel")
    out.append(f"  __host__ __device__ static constexpr int P(int l3) {{ constexpr int t[{lmax + 1}] = {{{', '.join(str(len(r)) for r in by_rank)}}}; return t[l3]; }}")
    out.append(f"  __host__ __device__ static constexpr int off(int l3) {{ constexpr int t[{lmax + 1}] = {{{', '.join(map(str, offs))}}}; return t[l3]; }}")
    out.append("};")
    out.append(f"__device__ __forceinline__ void ladder_t_{lmax}(const float (&b)[{D}], const float (&a)[{D}], float (&t)[{nt}]) {{")
    for l3 in range(lmax + 1):
        for j, p in enumerate(by_rank[l3]):
            l1, l2, _ = paths[p]
            out.append(f"  {{ // path {p}: ({l1},{l2},{l3})")
            for m3 in range(2 * l3 + 1):
                row = [(m1, terms) for (a3, m1, terms) in ent[p] if a3 == m3]
                dst = f"t[{offs[l3] + m3 * len(by_rank[l3]) + j}]"
                if not row:
                    out.append(f"    {dst} = 0.0f;")
                    continue
                first = True
                for m1, terms in row:
                    mexpr = " + ".join(f"{repr_f32(np.float32(v))}*a[{i}]" for v, i in terms)
                    if first:
                        out.append(f"    float s{m3} = ({mexpr}) * b[{idx(l1, m1 - l1)}];")
                        first = False
                    else:
                        out.append(f"    s{m3} = fmaf({mexpr}, b[{idx(l1, m1 - l1)}], s{m3});")
                out.append(f"    {dst} = s{m3};")
            out.append("  }")
    out.append("}")


# ---------------------------------------------------------------- per-path M entries

def path_m_entries(lmax):
    """Per path: the (m3, m1, terms) nonzeros of M in the order the code generator uses."""
    out = []
    for (l1, l2, l3) in paths_for(lmax):
        c = real_cg(l1, l2, l3)
        ent = []
        for m3 in range(2 * l3 + 1):
            for m1 in range(2 * l1 + 1):
                terms = [(c[m1, m2, m3], idx(l2, m2 - l2)) for m2 in range(2 * l2 + 1) if c[m1, m2, m3] != 0.0]
                if terms:
                    ent.append((m3, m1, terms))
        out.append(ent)
    return out


# ---------------------------------------------------------------- channel-major forward, path subsets

CX_LMAX = (1, 2)


def cx_subsets(lmax):
    """The two path subsets of the channel-major forward: subset 0 holds the paths with l1 < lmax,
    subset 1 those with l1 = lmax. Splitting by l1 means the warps of the two subsets read disjoint
    components of a sender row, so no component is loaded twice."""
    paths = paths_for(lmax)
    return [[p for p, t in enumerate(paths) if t[0] < lmax], [p for p, t in enumerate(paths) if t[0] == lmax]]


def cx_coefficients(lmax, subset):
    """Unique per-edge coefficients of a subset. Every nonzero M[m3][m1] = sum_m2 C Y[l2 m2] of a
    path with l2 > 0 is a fixed combination of one rank's harmonics; entries whose combinations agree
    up to sign share one stored value. Returns (keys, entry map): keys[i] = (l2, canonical vector),
    entry map[(p, m3, m1)] = (coefficient index, sign)."""
    paths = paths_for(lmax)
    ent = path_m_entries(lmax)
    keys, emap = [], {}
    for p in subset:
        l1, l2, l3 = paths[p]
        if l2 == 0:
            continue
        for m3, m1, terms in ent[p]:
            vec = [0.0] * (2 * l2 + 1)
            for v, i in terms:
                vec[i - idx(l2, -l2)] = v
            first = next(v for v in vec if v != 0.0)
            sgn = 1.0 if first > 0 else -1.0
            key = (l2, tuple(round(sgn * v, 12) for v in vec))
            if key not in keys:
                keys.append(key)
            emap[(p, m3, m1)] = (keys.index(key), sgn)
    return keys, emap


def emit_cx(out, lmax):
    paths = paths_for(lmax)
    ent = path_m_entries(lmax)
    subsets = cx_subsets(lmax)
    for s, sub in enumerate(subsets):
        keys, emap = cx_coefficients(lmax, sub)
        nc = max(4, -(-len(keys) // 4) * 4)
        l1s = sorted({paths[p][0] for p in sub})
        xcomps = [idx(l1, m) for l1 in l1s for m in range(-l1, l1 + 1)]
        ocomps = sorted({idx(paths[p][2], m) for p in sub for m in range(-paths[p][2], paths[p][2] + 1)})
        xi = {c: i for i, c in enumerate(xcomps)}
        oi = {c: i for i, c in enumerate(ocomps)}
        fma = 0
        out.append(f"// ---- channel-major forward, l_max = {lmax}, subset {s}: paths {sub}")
        out.append(f"template <> struct CxSub<{lmax}, {s}> {{")
        out.append(f"  static constexpr int NP = {len(sub)};   // paths")
        out.append(f"  static constexpr int NC = {nc};   // stored coefficients per edge (multiple of 4)")
        out.append(f"  static constexpr int NX = {len(xcomps)};   // sender-row components read")
        out.append(f"  static constexpr int NO = {len(ocomps)};   // output components written")
        for name, lst in (("path", sub), ("xcomp", xcomps), ("ocomp", ocomps)):
            out.append(f"  __host__ __device__ static constexpr int {name}(int i) {{")
            out.append(f"    constexpr int t[{len(lst)}] = {{{', '.join(str(v) for v in lst)}}};")
            out.append("    return t[i];")
            out.append("  }")
        # setup side: the coefficients from the harmonics
        out.append(f"  __device__ __forceinline__ static void coef(const float* Y, float (&c)[{nc}]) {{")
        for i, (l2, vec) in enumerate(keys):
            terms = [f"{repr_f32(np.float32(v))}*Y[{idx(l2, m2 - l2)}]" for m2, v in enumerate(vec) if v != 0.0]
            out.append(f"    c[{i}] = {' + '.join(terms)};")
        for i in range(len(keys), nc):
            out.append(f"    c[{i}] = 0.0f;")
        out.append("  }")
        # consumer side: one edge, NSL channels per lane
        out.append("  template <int NSL>")
        out.append(f"  __device__ __forceinline__ static void fwd(const float4* __restrict__ cf, const float (&x)[NSL][{len(xcomps)}],")
        out.append(f"      const float (&w)[NSL][{len(sub)}], float (&acc)[NSL][{len(ocomps)}]) {{")
        for q in range(nc // 4):
            out.append(f"    const float4 c4_{q} = cf[{q}];")
        out.append(f"    const float cv[{nc}] = {{" + ", ".join(f"c4_{q // 4}.{'xyzw'[q % 4]}" for q in range(nc)) + "};")
        out.append("    #pragma unroll")
        out.append("    for (int k = 0; k < NSL; ++k) {")
        for pi, p in enumerate(sub):
            l1, l2, l3 = paths[p]
            e = ent[p]
            out.append(f"      {{ // path {p}: ({l1},{l2},{l3})")
            out.append(f"        const float wp = w[k][{pi}];")
            if l2 == 0:
                for m3, m1, terms in e:
                    assert m3 == m1 and len(terms) == 1 and abs(terms[0][0] - 1.0) < 1e-12
                    o, xx = oi[idx(l3, m3 - l3)], xi[idx(l1, m1 - l1)]
                    out.append(f"        acc[k][{o}] = fmaf(wp, x[k][{xx}], acc[k][{o}]);")
                    fma += 1
            elif (2 * l1 + 1) < (2 * l3 + 1):
                for m1 in range(2 * l1 + 1):
                    out.append(f"        const float xs{m1} = wp * x[k][{xi[idx(l1, m1 - l1)]}];")
                    fma += 1
                for m3, m1, _ in e:
                    ci, sg = emap[(p, m3, m1)]
                    o = oi[idx(l3, m3 - l3)]
                    cexpr = f"cv[{ci}]" if sg > 0 else f"-cv[{ci}]"
                    out.append(f"        acc[k][{o}] = fmaf({cexpr}, xs{m1}, acc[k][{o}]);")
                    fma += 1
            else:
                for m3 in range(2 * l3 + 1):
                    row = [(a, m1) for (a, m1, _) in e if a == m3]
                    if not row:
                        continue
                    o = oi[idx(l3, m3 - l3)]
                    for j, (a, m1) in enumerate(row):
                        ci, sg = emap[(p, a, m1)]
                        cexpr = f"cv[{ci}]" if sg > 0 else f"-cv[{ci}]"
                        xv = f"x[k][{xi[idx(l1, m1 - l1)]}]"
                        if j == 0:
                            out.append(f"        float s{m3} = {cexpr} * {xv};")
                        else:
                            out.append(f"        s{m3} = fmaf({cexpr}, {xv}, s{m3});")
                        fma += 1
                    out.append(f"        acc[k][{o}] = fmaf(wp, s{m3}, acc[k][{o}]);")
                    fma += 1
            out.append("      }")
        out.append("    }")
        out.append("  }")
        out.append(f"  static constexpr int FMA = {fma};   // FP32 instructions per edge and channel")
        emit_cx_pair(out, sub, paths, ent, emap, nc, xi, oi)
        emit_cx_gw_pair(out, sub, paths, ent, emap, nc, xi, oi)
        out.append("};")


def emit_cx_pair(out, sub, paths, ent, emap, nc, xi, oi):
    """The same contraction for two edges of one receiver at once, in packed FP32 (f32x2) arithmetic:
    component .x belongs to the first edge, .y to the second. The coefficient row holds the two
    edges' coefficients interleaved (coefficient k of edge t at float 2 k + t). A coefficient used
    with a minus sign multiplies the negated x (exact), so each component sees exactly the roundings
    of the one-edge code."""
    nx, npth, no = len(xi), len(sub), len(oi)
    body, neg = [], set()
    for pi, p in enumerate(sub):
        l1, l2, l3 = paths[p]
        e = ent[p]
        body.append(f"    {{ // path {p}: ({l1},{l2},{l3})")
        if l2 == 0:
            for m3, m1, terms in e:
                o, xx = oi[idx(l3, m3 - l3)], xi[idx(l1, m1 - l1)]
                body.append(f"      acc[{o}] = __ffma2_rn(w[{pi}], x[{xx}], acc[{o}]);")
        elif (2 * l1 + 1) < (2 * l3 + 1):
            sgn = {}
            for m3, m1, _ in e:
                ci, sg = emap[(p, m3, m1)]
                sgn.setdefault(m1, set()).add(sg)
            for m1 in range(2 * l1 + 1):
                xx = xi[idx(l1, m1 - l1)]
                if 1 in sgn.get(m1, ()):
                    body.append(f"      const float2 xs{m1} = __fmul2_rn(w[{pi}], x[{xx}]);")
                if -1 in sgn.get(m1, ()):
                    neg.add(xx)
                    body.append(f"      const float2 xn{m1} = __fmul2_rn(w[{pi}], xm[{xx}]);")
            for m3, m1, _ in e:
                ci, sg = emap[(p, m3, m1)]
                o = oi[idx(l3, m3 - l3)]
                src = f"xs{m1}" if sg > 0 else f"xn{m1}"
                body.append(f"      acc[{o}] = __ffma2_rn(cv[{ci}], {src}, acc[{o}]);")
        else:
            for m3 in range(2 * l3 + 1):
                row = [(a, m1) for (a, m1, _) in e if a == m3]
                if not row:
                    continue
                o = oi[idx(l3, m3 - l3)]
                for j, (a, m1) in enumerate(row):
                    ci, sg = emap[(p, a, m1)]
                    xx = xi[idx(l1, m1 - l1)]
                    if sg < 0:
                        neg.add(xx)
                    xv = f"x[{xx}]" if sg > 0 else f"xm[{xx}]"
                    if j == 0:
                        body.append(f"      float2 s{m3} = __fmul2_rn(cv[{ci}], {xv});")
                    else:
                        body.append(f"      s{m3} = __ffma2_rn(cv[{ci}], {xv}, s{m3});")
                body.append(f"      acc[{o}] = __ffma2_rn(w[{pi}], s{m3}, acc[{o}]);")
        body.append("    }")
    out.append(f"  __device__ __forceinline__ static void fwd2(const float4* __restrict__ cf, const float2 (&x)[{nx}],")
    out.append(f"      const float2 (&w)[{npth}], float2 (&acc)[{no}]) {{")
    for q in range(nc // 2):
        out.append(f"    const float4 c4_{q} = cf[{q}];")
    out.append(f"    const float2 cv[{nc}] = {{" + ", ".join(
        f"make_float2(c4_{k // 2}.{'x' if k % 2 == 0 else 'z'}, c4_{k // 2}.{'y' if k % 2 == 0 else 'w'})" for k in range(nc)) + "};")
    if neg:
        out.append(f"    float2 xm[{nx}];")
        for xx in sorted(neg):
            out.append(f"    xm[{xx}] = __fmul2_rn(x[{xx}], make_float2(-1.0f, -1.0f));")
    out.extend(body)
    out.append("  }")


def emit_cx_gw_pair(out, sub, paths, ent, emap, nc, xi, oi):
    """Weight-gradient factor of the subset's paths for two edges at once (f32x2: .x the first edge,
    .y the second): gw_p = sum_{m1,m3} x[l1 m1] M_p[m3][m1] g[l3 m3], with M_p[m3][m1] = sum_m2 C Y
    from the pair-interleaved coefficient row. Each path contracts M with the longer side first
    (v = M^T g then x . v, or s = M x then g . s). A coefficient used with a minus sign multiplies
    the negated x or g (exact). sink(IC<p>{}, gw) receives path p (global path index)."""
    nx, no = len(xi), len(oi)
    body, negx, negg = [], set(), set()
    for pi, p in enumerate(sub):
        l1, l2, l3 = paths[p]
        e = ent[p]
        body.append(f"    {{ // path {p}: ({l1},{l2},{l3})")
        if l2 == 0:
            for j, (m3, m1, terms) in enumerate(e):
                o, xx = oi[idx(l3, m3 - l3)], xi[idx(l1, m1 - l1)]
                if j == 0:
                    body.append(f"      float2 t = __fmul2_rn(x[{xx}], g[{o}]);")
                else:
                    body.append(f"      t = __ffma2_rn(x[{xx}], g[{o}], t);")
            body.append(f"      sink(IC<{p}>{{}}, t);")
        elif (2 * l1 + 1) <= (2 * l3 + 1):
            # v[m1] = sum_m3 M[m3][m1] g[m3], then gw = sum_m1 x[m1] v[m1]
            first = True
            for m1 in range(2 * l1 + 1):
                col = [(m3, b) for (m3, b, _) in e if b == m1]
                if not col:
                    continue
                for j, (m3, _) in enumerate(col):
                    ci, sg = emap[(p, m3, m1)]
                    o = oi[idx(l3, m3 - l3)]
                    if sg < 0:
                        negg.add(o)
                    gv = f"g[{o}]" if sg > 0 else f"gm[{o}]"
                    if j == 0:
                        body.append(f"      float2 v{m1} = __fmul2_rn(cv[{ci}], {gv});")
                    else:
                        body.append(f"      v{m1} = __ffma2_rn(cv[{ci}], {gv}, v{m1});")
                xx = xi[idx(l1, m1 - l1)]
                if first:
                    body.append(f"      float2 t = __fmul2_rn(x[{xx}], v{m1});")
                    first = False
                else:
                    body.append(f"      t = __ffma2_rn(x[{xx}], v{m1}, t);")
            body.append(f"      sink(IC<{p}>{{}}, t);")
        else:
            # s[m3] = sum_m1 M[m3][m1] x[m1], then gw = sum_m3 g[m3] s[m3]
            first = True
            for m3 in range(2 * l3 + 1):
                row = [(a, m1) for (a, m1, _) in e if a == m3]
                if not row:
                    continue
                for j, (a, m1) in enumerate(row):
                    ci, sg = emap[(p, a, m1)]
                    xx = xi[idx(l1, m1 - l1)]
                    if sg < 0:
                        negx.add(xx)
                    xv = f"x[{xx}]" if sg > 0 else f"xm[{xx}]"
                    if j == 0:
                        body.append(f"      float2 s{m3} = __fmul2_rn(cv[{ci}], {xv});")
                    else:
                        body.append(f"      s{m3} = __ffma2_rn(cv[{ci}], {xv}, s{m3});")
                o = oi[idx(l3, m3 - l3)]
                if first:
                    body.append(f"      float2 t = __fmul2_rn(g[{o}], s{m3});")
                    first = False
                else:
                    body.append(f"      t = __ffma2_rn(g[{o}], s{m3}, t);")
            body.append(f"      sink(IC<{p}>{{}}, t);")
        body.append("    }")
    out.append("  template <class SINK>")
    out.append(f"  __device__ __forceinline__ static void gw2(const float4* __restrict__ cf, const float2 (&x)[{nx}],")
    out.append(f"      const float2 (&g)[{no}], SINK&& sink) {{")
    for q in range(nc // 2):
        out.append(f"    const float4 c4_{q} = cf[{q}];")
    out.append(f"    const float2 cv[{nc}] = {{" + ", ".join(
        f"make_float2(c4_{k // 2}.{'x' if k % 2 == 0 else 'z'}, c4_{k // 2}.{'y' if k % 2 == 0 else 'w'})" for k in range(nc)) + "};")
    if negx:
        out.append(f"    float2 xm[{nx}];")
        for xx in sorted(negx):
            out.append(f"    xm[{xx}] = __fmul2_rn(x[{xx}], make_float2(-1.0f, -1.0f));")
    if negg:
        out.append(f"    float2 gm[{no}];")
        for o in sorted(negg):
            out.append(f"    gm[{o}] = __fmul2_rn(g[{o}], make_float2(-1.0f, -1.0f));")
    out.extend(body)
    out.append("  }")


# ---------------------------------------------------------------- general irreps

GEN_LMAX = 4


def gen_triples():
    return [(a, b, c) for a in range(GEN_LMAX + 1) for b in range(GEN_LMAX + 1)
            for c in range(abs(a - b), min(GEN_LMAX, a + b) + 1)]


def emit_general(out):
    """Per coupling t = (l1, l2, l3): gbwd_t accumulates grad_x, dL/dY and dL/dw for one channel
    and one edge, gfwdc_t adds sum_edges w sum C Y x over a chunk of staged edges into
    acc[m3 * stride]. x, g and acc point at the channel's element of component 0 of their block;
    components are `stride` floats apart."""
    tri = gen_triples()
    out.append(f"constexpr int kGenLmax = {GEN_LMAX};")
    out.append(f"constexpr int kGenTriples = {len(tri)};")
    ids = [[[-1] * (GEN_LMAX + 1) for _ in range(GEN_LMAX + 1)] for _ in range(GEN_LMAX + 1)]
    for t, (a, b, c) in enumerate(tri):
        ids[a][b][c] = t
    flat = [ids[a][b][c] for a in range(GEN_LMAX + 1) for b in range(GEN_LMAX + 1) for c in range(GEN_LMAX + 1)]
    out.append("// coupling index of (l1, l2, l3) at [(l1 * 5 + l2) * 5 + l3], -1 outside the triangle rule")
    out.append("constexpr int kGenTriId[] = {" + ", ".join(map(str, flat)) + "};")
    nnz = [int(np.count_nonzero(real_cg_any(*t))) for t in tri]
    out.append("constexpr int kGenTriNnz[] = {" + ", ".join(map(str, nnz)) + "};")
    for t, (l1, l2, l3) in enumerate(tri):
        c = real_cg_any(l1, l2, l3)
        groups = []   # (m3, m1, [(coef, y index)])
        for m3 in range(2 * l3 + 1):
            for m1 in range(2 * l1 + 1):
                terms = [(c[m1, m2, m3], idx(l2, m2 - l2)) for m2 in range(2 * l2 + 1) if c[m1, m2, m3] != 0.0]
                if terms:
                    groups.append((m3, m1, terms))
        out.append(f"// ({l1},{l2},{l3})")
        # backward
        out.append("template <int S>   // S: the block stride when known at compile time (0: stride_rt)")
        out.append(f"__device__ __forceinline__ void gbwd_{t}(const float* __restrict__ x, const float* __restrict__ g,")
        out.append("                                       int stride_rt, const float* Y, float w, float* gx, float* gY,")
        out.append("                                       float& gw) {")
        out.append("  const int stride = S ? S : stride_rt;")
        for m1 in range(2 * l1 + 1):
            out.append(f"  const float x{m1} = x[{m1} * stride];")
            out.append(f"  float a{m1} = 0.0f;")
        for m3 in range(2 * l3 + 1):
            out.append(f"  const float g{m3} = g[{m3} * stride];")
        # dL/dY_i = w sum_terms C x g: the sums over the coupling's terms first, one product with w
        # per harmonic component at the end
        ys = sorted({i for _, _, terms in groups for _, i in terms})
        for i in ys:
            out.append(f"  float t{i} = 0.0f;")
        # two equivalent orders, the one with fewer operations is emitted:
        #   A: mv = sum C Y per (m3, m1), a += mv g, xg = x g, t_i += C xg
        #   B: cg = C g per (C, m3), then per term a += Y cg and t_i += x cg
        cost_a = len({tuple(terms) for _, _, terms in groups}) + 2 * len(groups) + sum(len(t) for _, _, t in groups)
        cost_b = len({(np.float32(v), m3) for m3, _, terms in groups for v, _ in terms}) + \
            2 * sum(len(t) for _, _, t in groups)
        for m3, m1, terms in groups:
            if cost_a <= cost_b:
                mexpr = " + ".join(f"{repr_f32(np.float32(v))}*Y[{i}]" for v, i in terms)
                out.append(f"  {{ const float mv = {mexpr};")
                out.append(f"    a{m1} = fmaf(mv, g{m3}, a{m1});")
                out.append(f"    const float xg = x{m1} * g{m3};")
                for v, i in terms:
                    out.append(f"    t{i} = fmaf({repr_f32(np.float32(v))}, xg, t{i});")
                out.append("  }")
            else:
                for v, i in terms:
                    out.append(f"  {{ const float cg = {repr_f32(np.float32(v))} * g{m3};")
                    out.append(f"    a{m1} = fmaf(Y[{i}], cg, a{m1});")
                    out.append(f"    t{i} = fmaf(x{m1}, cg, t{i}); }}")
        for i in ys:
            out.append(f"  gY[{i}] = fmaf(w, t{i}, gY[{i}]);")
        # dL/dw = sum_{m1, m3} x M g = sum_m1 x[m1] a[m1]
        for m1 in range(2 * l1 + 1):
            out.append(f"  gw = fmaf(x{m1}, a{m1}, gw);")
        for m1 in range(2 * l1 + 1):
            out.append(f"  gx[{m1} * stride] = fmaf(w, a{m1}, gx[{m1} * stride]);")
        out.append("}")
    # forward over a chunk of staged edges: the channel's path sums stay in registers across the
    # chunk, and the path's radial weights are projected per edge from the staged R
    out.append(f"constexpr int kGenGeoF = 33;   // staged floats per edge: Y (25), R (8)")
    for t, (l1, l2, l3) in enumerate(tri):
        c = real_cg_any(l1, l2, l3)
        groups = []
        for m3 in range(2 * l3 + 1):
            for m1 in range(2 * l1 + 1):
                terms = [(c[m1, m2, m3], idx(l2, m2 - l2)) for m2 in range(2 * l2 + 1) if c[m1, m2, m3] != 0.0]
                if terms:
                    groups.append((m3, m1, terms))
        out.append(f"__device__ __forceinline__ void gfwdc_{t}(const float* geo, const int* sj, int cnt,")
        out.append("                                        const float* __restrict__ xu, int dim_in, int stride,")
        out.append("                                        const float* wb, float* acc, const unsigned* mk, unsigned bit) {")
        rows = sorted({m3 for m3, _, _ in groups})
        for m3 in rows:
            out.append(f"  float a{m3} = 0.0f;")
        out.append("  for (int k = 0; k < cnt; ++k) {")
        out.append("    if (mk && !(mk[k] & bit)) continue;   // path off for this edge")
        out.append("    const float* Y = geo + k * kGenGeoF;")
        out.append("    float w = 0.0f;")
        out.append("    #pragma unroll")
        out.append("    for (int b = 0; b < 8; ++b) w = fmaf(Y[25 + b], wb[b], w);")
        out.append("    const float* x = xu + static_cast<size_t>(sj[k]) * dim_in;")
        for m1 in range(2 * l1 + 1):
            out.append(f"    const float x{m1} = x[{m1} * stride];")
        for m3 in rows:
            row = [(m1, terms) for (a3, m1, terms) in groups if a3 == m3]
            first = True
            for m1, terms in row:
                mexpr = " + ".join(f"{repr_f32(np.float32(v))}*Y[{i}]" for v, i in terms)
                if first:
                    out.append(f"    float s{m3} = ({mexpr}) * x{m1};")
                    first = False
                else:
                    out.append(f"    s{m3} = fmaf({mexpr}, x{m1}, s{m3});")
            out.append(f"    a{m3} = fmaf(w, s{m3}, a{m3});")
        out.append("  }")
        for m3 in rows:
            out.append(f"  acc[{m3} * stride] += a{m3};")
        out.append("}")
    # weight gradient over a chunk of staged edges: gw = sum_m3 g[m3] sum C Y x per edge, then
    # acc8[b] += R_b gw (the channel's column of dL/dW)
    for t, (l1, l2, l3) in enumerate(tri):
        c = real_cg_any(l1, l2, l3)
        groups = []
        for m3 in range(2 * l3 + 1):
            for m1 in range(2 * l1 + 1):
                terms = [(c[m1, m2, m3], idx(l2, m2 - l2)) for m2 in range(2 * l2 + 1) if c[m1, m2, m3] != 0.0]
                if terms:
                    groups.append((m3, m1, terms))
        rows = sorted({m3 for m3, _, _ in groups})
        out.append("template <int S>   // S: the block stride when known at compile time (0: stride_rt)")
        out.append(f"__device__ __forceinline__ void gdwc_{t}(const float* geo, const int* sj, const int* si, int cnt,")
        out.append("                                       const float* __restrict__ xu, const float* __restrict__ gu,")
        out.append("                                       int dim_in, int dim_out, int stride_rt, float* acc8) {")
        out.append("  const int stride = S ? S : stride_rt;")
        out.append("  for (int k = 0; k < cnt; ++k) {")
        out.append("    const float* Y = geo + k * kGenGeoF;")
        out.append("    const float* x = xu + static_cast<size_t>(sj[k]) * dim_in;")
        out.append("    const float* g = gu + static_cast<size_t>(si[k]) * dim_out;")
        for m1 in range(2 * l1 + 1):
            out.append(f"    const float x{m1} = x[{m1} * stride];")
        out.append("    float gw = 0.0f;")
        for m3 in rows:
            row = [(m1, terms) for (a3, m1, terms) in groups if a3 == m3]
            first = True
            for m1, terms in row:
                mexpr = " + ".join(f"{repr_f32(np.float32(v))}*Y[{i}]" for v, i in terms)
                if first:
                    out.append(f"    float s{m3} = ({mexpr}) * x{m1};")
                    first = False
                else:
                    out.append(f"    s{m3} = fmaf({mexpr}, x{m1}, s{m3});")
            out.append(f"    gw = fmaf(g[{m3} * stride], s{m3}, gw);")
        out.append("    #pragma unroll")
        out.append("    for (int b = 0; b < 8; ++b) acc8[b] = fmaf(Y[25 + b], gw, acc8[b]);")
        out.append("  }")
        out.append("}")
    out.append("__device__ __forceinline__ void gen_dw_chunk(int t, const float* geo, const int* sj, const int* si, int cnt,")
    out.append("                                             const float* xu, const float* gu, int dim_in, int dim_out,")
    out.append("                                             int stride, float* acc8) {")
    out.append("  switch (t) {")
    for t in range(len(tri)):
        out.append(f"    case {t}:")
        for st in (32, 64, 128):
            kw = "if" if st == 32 else "else if"
            out.append(f"      {kw} (stride == {st}) gdwc_{t}<{st}>(geo, sj, si, cnt, xu, gu, dim_in, dim_out, stride, acc8);")
        out.append(f"      else gdwc_{t}<0>(geo, sj, si, cnt, xu, gu, dim_in, dim_out, stride, acc8);")
        out.append("      break;")
    out.append("    default: break;")
    out.append("  }")
    out.append("}")
    # forward over a round of staged edges with the radial weights supplied: wl(k0, w) fills w[0..3]
    # with the channel's weights of edges k0..k0+3 (warp-uniform call); the edges run in quads with
    # all their loads ahead of the arithmetic (the caller pads the round to whole quads with edges
    # of zero weight and zero harmonics). Instantiated for the block strides 32, 64 and 128
    # (component loads at immediate offsets) and for any stride.
    out.append("constexpr int kGenYS = 25;   // staged harmonics per edge (to l = 4)")
    for t, (l1, l2, l3) in enumerate(tri):
        c = real_cg_any(l1, l2, l3)
        groups = []
        for m3 in range(2 * l3 + 1):
            for m1 in range(2 * l1 + 1):
                terms = [(c[m1, m2, m3], idx(l2, m2 - l2)) for m2 in range(2 * l2 + 1) if c[m1, m2, m3] != 0.0]
                if terms:
                    groups.append((m3, m1, terms))
        rows = sorted({m3 for m3, _, _ in groups})

        def body(ind, k, w):
            lines = [f"{ind}{{ const float* Y = Ys + ({k}) * kGenYS;",
                     f"{ind}  const float* x = xu + static_cast<size_t>(sj[{k}]) * dim_in;"]
            for m1 in range(2 * l1 + 1):
                lines.append(f"{ind}  const float x{m1} = x[{m1} * stride];")
            for m3 in rows:
                row = [(m1, terms) for (a3, m1, terms) in groups if a3 == m3]
                first = True
                for m1, terms in row:
                    mexpr = " + ".join(f"{repr_f32(np.float32(v))}*Y[{i}]" for v, i in terms)
                    if first:
                        lines.append(f"{ind}  float s{m3} = ({mexpr}) * x{m1};")
                        first = False
                    else:
                        lines.append(f"{ind}  s{m3} = fmaf({mexpr}, x{m1}, s{m3});")
                lines.append(f"{ind}  a{m3} = fmaf({w}, s{m3}, a{m3});")
            lines.append(f"{ind}}}")
            return lines

        out.append("template <int S, class WL>   // S: the block stride when known at compile time (0: stride_rt)")
        out.append(f"__device__ __forceinline__ void gfwdw_{t}(const float* Ys, const int* sj, int cnt,")
        out.append("                                        const float* __restrict__ xu, int dim_in, int stride_rt, WL&& wl,")
        out.append("                                        bool act, float* acc) {")
        out.append("  const int stride = S ? S : stride_rt;")
        for m3 in rows:
            out.append(f"  float a{m3} = 0.0f;")
        out.append("  for (int k0 = 0; k0 < cnt; k0 += 4) {   // cnt: a multiple of 4 (padding edges weigh zero)")
        out.append("    float w[4];")
        out.append("    wl(k0, w);")
        out.append("    if (act) {")
        out.append("      #pragma unroll")
        out.append("      for (int kk = 0; kk < 4; ++kk)")
        out.extend(body("        ", "k0 + kk", "w[kk]"))
        out.append("    }")
        out.append("  }")
        out.append("  if (act) {")
        for m3 in rows:
            out.append(f"    acc[{m3} * stride] += a{m3};")
        out.append("  }")
        out.append("}")
    out.append("template <class WL>")
    out.append("__device__ __forceinline__ void gen_fwd_w(int t, const float* Ys, const int* sj, int cnt, const float* xu,")
    out.append("                                          int dim_in, int stride, WL&& wl, bool act, float* acc) {")
    out.append("  switch (t) {")
    for t in range(len(tri)):
        out.append(f"    case {t}:")
        for st in (32, 64, 128):
            kw = "if" if st == 32 else "else if"
            out.append(f"      {kw} (stride == {st}) gfwdw_{t}<{st}>(Ys, sj, cnt, xu, dim_in, stride, wl, act, acc);")
        out.append(f"      else gfwdw_{t}<0>(Ys, sj, cnt, xu, dim_in, stride, wl, act, acc);")
        out.append("      break;")
    out.append("    default: break;")
    out.append("  }")
    out.append("}")
    out.append("// mk: per-edge path masks of the chunk (null: every path on); bit: this path's bit")
    out.append("__device__ __forceinline__ void gen_fwd_chunk(int t, const float* geo, const int* sj, int cnt,")
    out.append("                                              const float* xu, int dim_in, int stride, const float* wb,")
    out.append("                                              float* acc, const unsigned* mk, unsigned bit) {")
    out.append("  switch (t) {")
    for t in range(len(tri)):
        out.append(f"    case {t}: gfwdc_{t}(geo, sj, cnt, xu, dim_in, stride, wb, acc, mk, bit); break;")
    out.append("    default: break;")
    out.append("  }")
    out.append("}")
    out.append("__device__ __forceinline__ void gen_bwd(int t, const float* x, const float* g, int stride, const float* Y,")
    out.append("                                        float w, float* gx, float* gY, float& gw) {")
    out.append("  switch (t) {")
    for t in range(len(tri)):
        out.append(f"    case {t}:")
        for st in (32, 64, 128):
            kw = "if" if st == 32 else "else if"
            out.append(f"      {kw} (stride == {st}) gbwd_{t}<{st}>(x, g, stride, Y, w, gx, gY, gw);")
        out.append(f"      else gbwd_{t}<0>(x, g, stride, Y, w, gx, gY, gw);")
        out.append("      break;")
    out.append("    default: break;")
    out.append("  }")
    out.append("}")


def generate():
    out = ["// GENERATED by gen_paths.py -- do not edit.",
           "// Real-basis Clebsch-Gordan contractions and real spherical harmonics, unrolled per path.",
           "#pragma once",
           "#include <type_traits>",
           "namespace etp_gen {",
           "// compile-time path index handed to the weight-fetch callback",
           "template <int N> struct IC {",
           "  static constexpr int value = N;",
           "  __host__ __device__ constexpr operator int() const { return N; }",
           "};",
           "// wfetch(IC<p>, w...) fills the path's weights; a callback that returns bool can skip the",
           "// path (false: no contribution), one that returns nothing always computes it",
           "template <class F, class... A>",
           "__device__ __forceinline__ bool fetch(F&& f, A&&... a) {",
           "  if constexpr (std::is_void_v<decltype(f(a...))>) {",
           "    f(a...);",
           "    return true;",
           "  } else {",
           "    return f(a...);",
           "  }",
           "}",
           "template <int L> struct PathSet;",
           "template <int L, int S> struct CxSub;",
           "template <int L> struct LadderShape;"]
    for lmax in LMAX_SUPPORTED:
        emit_sh(out, lmax)
        emit_paths(out, lmax)
    for lmax in CX_LMAX:
        emit_cx(out, lmax)
    for lmax in LMAX_SUPPORTED:
        emit_node(out, lmax)
        emit_ladder_t(out, lmax)
    emit_sh(out, GEN_LMAX)
    emit_general(out)
    out.append("}  // namespace etp_gen")
    return "\n".join(out) + "\n"


if __name__ == "__main__":
    dst = os.path.join(HERE, "generated", "etp_paths.h")
    os.makedirs(os.path.dirname(dst), exist_ok=True)
    text = generate()
    if len(sys.argv) > 1 and sys.argv[1] == "--check":
        sys.exit(0 if os.path.exists(dst) and open(dst).read() == text else 1)
    with open(dst, "w") as f:
        f.write(text)
    print("wrote", dst)
