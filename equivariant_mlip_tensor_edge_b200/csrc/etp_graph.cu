// Graph construction: brute-force neighbour list with a fixed float64 inclusion test, canonical
// receiver-sorted CSR, and the transposed (sender-sorted) order. Integer outputs are
// deterministic and bit-exact against any implementation of the same test (include/etp.h).
#include <cub/cub.cuh>

#include <cmath>
#include <cstdlib>
#include <string>

#include "etp_internal.h"

namespace etp {
namespace {

struct CellParams {
  double c[9];       // rows = lattice vectors
  int n[3];          // images scanned per axis: S_a in [-n_a, n_a]
  double rc2;        // float64(r_cut)^2 (exact: a float squared fits in a double)
  // Orthorhombic cell whose periodic lengths all exceed 2 r_cut: two images of a pair differ by
  // more than 2 r_cut along some axis, so at most one image can be within r_cut and it is the
  // nearest one. Testing only that image (clamped to the scanned range) keeps exactly the set of
  // edges the full scan keeps, with the same arithmetic for the kept edge.
  int min_image;
  double len[3];
};

// r = (pos[j] - pos[i]) + ((S0 c0 + S1 c1) + S2 c2); d2 = (rx rx + ry ry) + rz rz, no FMA.
__device__ __forceinline__ bool pair_test(float3 pi, float3 pj, int s0, int s1, int s2,
                                          const CellParams& cp, double* rx, double* ry, double* rz) {
  const double a0 = static_cast<double>(s0), a1 = static_cast<double>(s1), a2 = static_cast<double>(s2);
  const double sx = __dadd_rn(__dadd_rn(__dmul_rn(a0, cp.c[0]), __dmul_rn(a1, cp.c[3])), __dmul_rn(a2, cp.c[6]));
  const double sy = __dadd_rn(__dadd_rn(__dmul_rn(a0, cp.c[1]), __dmul_rn(a1, cp.c[4])), __dmul_rn(a2, cp.c[7]));
  const double sz = __dadd_rn(__dadd_rn(__dmul_rn(a0, cp.c[2]), __dmul_rn(a1, cp.c[5])), __dmul_rn(a2, cp.c[8]));
  const double dx = __dadd_rn(__dsub_rn(static_cast<double>(pj.x), static_cast<double>(pi.x)), sx);
  const double dy = __dadd_rn(__dsub_rn(static_cast<double>(pj.y), static_cast<double>(pi.y)), sy);
  const double dz = __dadd_rn(__dsub_rn(static_cast<double>(pj.z), static_cast<double>(pi.z)), sz);
  const double d2 = __dadd_rn(__dadd_rn(__dmul_rn(dx, dx), __dmul_rn(dy, dy)), __dmul_rn(dz, dz));
  *rx = dx;
  *ry = dy;
  *rz = dz;
  return d2 < cp.rc2;
}

__device__ __forceinline__ float3 load_pos(const float* pos, int i) {
  return make_float3(pos[3 * i], pos[3 * i + 1], pos[3 * i + 2]);
}

__device__ __forceinline__ int nearest_image(float pi, float pj, double len, int n) {
  if (n == 0) return 0;
  const double d = static_cast<double>(pj) - static_cast<double>(pi);
  int k = -static_cast<int>(rint(d / len));
  return k < -n ? -n : (k > n ? n : k);
}

// Number of kept images for receiver i and sender j (S in lexicographic order).
__device__ __forceinline__ int count_pair(float3 pi, float3 pj, bool same, const CellParams& cp) {
  int c = 0;
  double rx, ry, rz;
  if (cp.min_image) {
    const int s0 = nearest_image(pi.x, pj.x, cp.len[0], cp.n[0]);
    const int s1 = nearest_image(pi.y, pj.y, cp.len[1], cp.n[1]);
    const int s2 = nearest_image(pi.z, pj.z, cp.len[2], cp.n[2]);
    if (same && s0 == 0 && s1 == 0 && s2 == 0) return 0;
    return pair_test(pi, pj, s0, s1, s2, cp, &rx, &ry, &rz) ? 1 : 0;
  }
  for (int s0 = -cp.n[0]; s0 <= cp.n[0]; ++s0)
    for (int s1 = -cp.n[1]; s1 <= cp.n[1]; ++s1)
      for (int s2 = -cp.n[2]; s2 <= cp.n[2]; ++s2) {
        if (same && s0 == 0 && s1 == 0 && s2 == 0) continue;
        c += pair_test(pi, pj, s0, s1, s2, cp, &rx, &ry, &rz) ? 1 : 0;
      }
  return c;
}

constexpr int kChunk = 256;   // senders per warp task

// One warp per (receiver i, chunk c of kChunk senders): counts[i * n_chunks + c] = kept pairs.
__global__ void k_nbr_count(const float* __restrict__ pos, int n, int n_chunks, CellParams cp,
                            int* __restrict__ counts) {
  const int lane = threadIdx.x & 31;
  const long long n_tasks = static_cast<long long>(n) * n_chunks;
  const long long stride = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long t = blockIdx.x * static_cast<long long>(blockDim.x >> 5) + (threadIdx.x >> 5); t < n_tasks;
       t += stride) {
    const int i = static_cast<int>(t / n_chunks);
    const int j_beg = static_cast<int>(t % n_chunks) * kChunk;
    const int j_end = j_beg + kChunk < n ? j_beg + kChunk : n;
    const float3 pi = load_pos(pos, i);
    int c = 0;
    for (int j = j_beg + lane; j < j_end; j += 32) c += count_pair(pi, load_pos(pos, j), j == i, cp);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (lane == 0) counts[t] = c;
  }
}

// row_ptr[0] = 0, row_ptr[i + 1] = inclusive chunk sum at the last chunk of receiver i.
__global__ void k_row_ptr_chunks(const int* __restrict__ incl, int n, int n_chunks, int* __restrict__ row_ptr) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i <= n; i += gridDim.x * blockDim.x)
    row_ptr[i] = i == 0 ? 0 : incl[static_cast<long long>(i) * n_chunks - 1];
}

// One warp per (receiver, chunk): writes the chunk's pairs in canonical (sender, S) order at the
// chunk's offset (exclusive chunk sum), and the receiver of every written edge.
__global__ void k_nbr_emit(const float* __restrict__ pos, int n, int n_chunks, CellParams cp,
                           const int* __restrict__ counts, const int* __restrict__ incl,
                           int* __restrict__ sender, float* __restrict__ edge_vec, int* __restrict__ shift,
                           int* __restrict__ receiver) {
  const int lane = threadIdx.x & 31;
  const long long n_tasks = static_cast<long long>(n) * n_chunks;
  const long long stride = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long t = blockIdx.x * static_cast<long long>(blockDim.x >> 5) + (threadIdx.x >> 5); t < n_tasks;
       t += stride) {
    if (counts[t] == 0) continue;
    const int i = static_cast<int>(t / n_chunks);
    const int j_beg = static_cast<int>(t % n_chunks) * kChunk;
    const int j_end = j_beg + kChunk < n ? j_beg + kChunk : n;
    const float3 pi = load_pos(pos, i);
    int base = incl[t] - counts[t];
    for (int j0 = j_beg; j0 < j_end; j0 += 32) {
      const int j = j0 + lane;
      const float3 pj = j < j_end ? load_pos(pos, j) : pi;
      const int c = j < j_end ? count_pair(pi, pj, j == i, cp) : 0;
      int incl_c = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl_c, o);
        if (lane >= o) incl_c += v;
      }
      const int total = __shfl_sync(0xffffffffu, incl_c, 31);
      if (c > 0 && cp.min_image) {
        const int s0 = nearest_image(pi.x, pj.x, cp.len[0], cp.n[0]);
        const int s1 = nearest_image(pi.y, pj.y, cp.len[1], cp.n[1]);
        const int s2 = nearest_image(pi.z, pj.z, cp.len[2], cp.n[2]);
        double rx, ry, rz;
        pair_test(pi, pj, s0, s1, s2, cp, &rx, &ry, &rz);
        const int at = base + incl_c - c;
        sender[at] = j;
        receiver[at] = i;
        edge_vec[3 * at + 0] = static_cast<float>(rx);
        edge_vec[3 * at + 1] = static_cast<float>(ry);
        edge_vec[3 * at + 2] = static_cast<float>(rz);
        if (shift) {
          shift[3 * at + 0] = s0;
          shift[3 * at + 1] = s1;
          shift[3 * at + 2] = s2;
        }
      } else if (c > 0) {
        int at = base + incl_c - c;
        double rx, ry, rz;
        for (int s0 = -cp.n[0]; s0 <= cp.n[0]; ++s0)
          for (int s1 = -cp.n[1]; s1 <= cp.n[1]; ++s1)
            for (int s2 = -cp.n[2]; s2 <= cp.n[2]; ++s2) {
              if (j == i && s0 == 0 && s1 == 0 && s2 == 0) continue;
              if (pair_test(pi, pj, s0, s1, s2, cp, &rx, &ry, &rz)) {
                sender[at] = j;
                receiver[at] = i;
                edge_vec[3 * at + 0] = static_cast<float>(rx);
                edge_vec[3 * at + 1] = static_cast<float>(ry);
                edge_vec[3 * at + 2] = static_cast<float>(rz);
                if (shift) {
                  shift[3 * at + 0] = s0;
                  shift[3 * at + 1] = s1;
                  shift[3 * at + 2] = s2;
                }
                ++at;
              }
            }
      }
      base += total;
    }
  }
}

// ------------------------------------------------------------------ cell binning
// The binned search finds the same edge set as the all-pairs scan above: it only narrows the
// candidates (j, S) that reach pair_test. Atoms are binned by fractional coordinate
// f = pos inv(cell) (Cartesian coordinates when there is no cell). Periodic axis a: nb_a bins of
// width 1 / nb_a in f, i.e. at least r_cut (1 + 1e-6) along the plane normal; an atom's bin is
// floor((f - floor f) nb_a) and its wrap count floor f. Non-periodic axis: bins of width
// r_cut (1 + 1e-6) / spacing_a in f, bin floor(f / width). Two points within r_cut differ by less
// than r_cut / spacing_a in f_a, so their bins differ by at most K_a on every axis; the candidates
// of receiver i are the atoms of the bins b_i + d, |d_a| <= K_a, with image S_a = q_a + w_i - w_j
// (q_a: the wrap of b_i + d on a periodic axis, 0 otherwise), kept iff |S_a| <= n_a and the exact
// pair_test passes. Each kept pair then goes to its rank by (sender, S) within the row, which is
// the canonical order.
struct BinParams {
  double inv[9];     // f_a = sum_k pos_k inv[3 k + a]
  int periodic[3];
  int nb[3];         // periodic axes: bins per axis
  double width[3];   // non-periodic axes: bin width in f
  int K[3];          // bin offsets scanned per axis: d_a in [-K_a, K_a]
  int n_off;         // (2 K0 + 1)(2 K1 + 1)(2 K2 + 1)
  long long n_s;     // images per sender: (2 n0 + 1)(2 n1 + 1)(2 n2 + 1)
};

constexpr int kBinBias = 1 << 20;           // bin coordinates are stored biased, in 21 bits
constexpr unsigned long long kBinMask = (1ull << 21) - 1;

__device__ __forceinline__ unsigned long long bin_key(int b0, int b1, int b2) {
  return (static_cast<unsigned long long>(b0 + kBinBias) << 42) |
         (static_cast<unsigned long long>(b1 + kBinBias) << 21) | static_cast<unsigned long long>(b2 + kBinBias);
}

__device__ __forceinline__ int key_coord(unsigned long long key, int a) {
  return static_cast<int>((key >> (21 * (2 - a))) & kBinMask) - kBinBias;
}

// Per atom: its bin key (this unsorted array also serves the receiver side), the atom id, its wrap
// counts.
// flag bit 0: a coordinate outside the representable bin range (the caller then scans all pairs).
__global__ void k_bin_atoms(const float* __restrict__ pos, int n, BinParams bp, unsigned long long* __restrict__ key,
                            int* __restrict__ atom, int* __restrict__ wrap, int* __restrict__ flag) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const double p[3] = {static_cast<double>(pos[3 * i]), static_cast<double>(pos[3 * i + 1]),
                         static_cast<double>(pos[3 * i + 2])};
    int b[3];
    for (int a = 0; a < 3; ++a) {
      const double f = (p[0] * bp.inv[a] + p[1] * bp.inv[3 + a]) + p[2] * bp.inv[6 + a];
      int w = 0, bb;
      if (bp.periodic[a]) {
        const double fl = floor(f);
        const bool fits = fabs(fl) < 1.0e8;   // wrap counts and their differences stay ints
        if (!fits) atomicOr(flag, 1);
        w = fits ? static_cast<int>(fl) : 0;
        bb = static_cast<int>(floor((f - fl) * bp.nb[a]));
        bb = bb < 0 ? 0 : (bb >= bp.nb[a] ? bp.nb[a] - 1 : bb);
      } else {
        const double q = floor(f / bp.width[a]);
        if (!(fabs(q) < static_cast<double>(kBinBias - 4))) {
          atomicOr(flag, 1);
          bb = 0;
        } else {
          bb = static_cast<int>(q);
        }
      }
      b[a] = bb;
      wrap[3 * i + a] = w;
    }
    const unsigned long long k = bin_key(b[0], b[1], b[2]);
    key[i] = k;
    atom[i] = i;
  }
}

__device__ __forceinline__ int lower_bound_u64(const unsigned long long* __restrict__ v, int n, unsigned long long x) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (v[mid] < x) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// One warp per receiver. EMIT = false: counts[i] = kept pairs. EMIT = true: the row's keys
// (sender * n_s + image index) are first written in bin order to the row's slots of `ekey`; then
// every key goes to its canonical place, base + (number of smaller keys in the row), where its
// sender, image and r (recomputed by the same pair_test) are stored, with the receiver.
template <bool EMIT>
__global__ void k_bin_pairs(const float* __restrict__ pos, int n, CellParams cp, BinParams bp,
                            const unsigned long long* __restrict__ skey, const int* __restrict__ satom,
                            const unsigned long long* __restrict__ akey, const int* __restrict__ wrap,
                            int* __restrict__ counts, const int* __restrict__ row_ptr,
                            unsigned long long* __restrict__ ekey, int* __restrict__ receiver,
                            int* __restrict__ sender, float* __restrict__ edge_vec, int* __restrict__ shift) {
  const int lane = threadIdx.x & 31;
  const int stride = gridDim.x * (blockDim.x >> 5);
  for (int i = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); i < n; i += stride) {
    const float3 pi = load_pos(pos, i);
    const unsigned long long ki = akey[i];
    const int bi[3] = {key_coord(ki, 0), key_coord(ki, 1), key_coord(ki, 2)};
    const int wi[3] = {wrap[3 * i], wrap[3 * i + 1], wrap[3 * i + 2]};
    int count = 0;
    const int base = EMIT ? row_ptr[i] : 0;
    const int row_end = EMIT ? row_ptr[i + 1] : 0;   // the count pass kept exactly this many
    for (int o0 = 0; o0 < bp.n_off; o0 += 32) {
      // lane o: the bin b_i + d of offset index o0 + lane, its atom range and wrap
      const int o = o0 + lane;
      bool have = o < bp.n_off;
      int lo = 0, hi = 0, q[3] = {0, 0, 0};
      if (have) {
        int rem = o, bb[3];
        for (int a = 2; a >= 0; --a) {
          const int span = 2 * bp.K[a] + 1;
          const int d = rem % span - bp.K[a];
          rem /= span;
          int u = bi[a] + d;
          if (bp.periodic[a]) {
            const int nb = bp.nb[a];
            const int qq = u >= 0 ? u / nb : -((-u + nb - 1) / nb);
            q[a] = qq;
            u -= qq * nb;
          } else if (u <= -kBinBias || u >= kBinBias) {
            have = false;
          }
          bb[a] = u;
        }
        if (have) {
          const unsigned long long kb = bin_key(bb[0], bb[1], bb[2]);
          lo = lower_bound_u64(skey, n, kb);
          hi = lower_bound_u64(skey, n, kb + 1);
        }
      }
      for (int src = 0; src < 32; ++src) {
        const int blo = __shfl_sync(0xffffffffu, lo, src);
        const int bhi = __shfl_sync(0xffffffffu, hi, src);
        const int q0 = __shfl_sync(0xffffffffu, q[0], src);
        const int q1 = __shfl_sync(0xffffffffu, q[1], src);
        const int q2 = __shfl_sync(0xffffffffu, q[2], src);
        for (int t = blo; t < bhi; t += 32) {
          const int idx = t + lane;
          bool keep = false;
          int j = 0, s0 = 0, s1 = 0, s2 = 0;
          if (idx < bhi) {
            j = satom[idx];
            s0 = bp.periodic[0] ? q0 + wi[0] - wrap[3 * j] : 0;
            s1 = bp.periodic[1] ? q1 + wi[1] - wrap[3 * j + 1] : 0;
            s2 = bp.periodic[2] ? q2 + wi[2] - wrap[3 * j + 2] : 0;
            keep = abs(s0) <= cp.n[0] && abs(s1) <= cp.n[1] && abs(s2) <= cp.n[2] &&
                   !(j == i && s0 == 0 && s1 == 0 && s2 == 0);
            if (keep) {
              double rx, ry, rz;
              keep = pair_test(pi, load_pos(pos, j), s0, s1, s2, cp, &rx, &ry, &rz);
            }
          }
          const unsigned m = __ballot_sync(0xffffffffu, keep);
          const int at = base + count + __popc(m & ((1u << lane) - 1u));
          if (EMIT && keep && at < row_end) {
            const long long sidx =
                (static_cast<long long>(s0 + cp.n[0]) * (2 * cp.n[1] + 1) + (s1 + cp.n[1])) * (2 * cp.n[2] + 1) +
                (s2 + cp.n[2]);
            ekey[at] = static_cast<unsigned long long>(j) * static_cast<unsigned long long>(bp.n_s) +
                       static_cast<unsigned long long>(sidx);
          }
          count += __popc(m);
        }
      }
    }
    if (!EMIT) {
      if (lane == 0) counts[i] = count;
      continue;
    }
    __syncwarp();   // the row's keys, written by every lane, are visible to the whole warp
    const int len = row_end - base;
    const int w2 = 2 * cp.n[2] + 1, w1 = 2 * cp.n[1] + 1;
    for (int t = lane; t < len; t += 32) {
      const unsigned long long key = ekey[base + t];
      int rank = 0;
      for (int u = 0; u < len; ++u) rank += ekey[base + u] < key ? 1 : 0;   // keys are distinct
      const int j = static_cast<int>(key / static_cast<unsigned long long>(bp.n_s));
      long long sidx = static_cast<long long>(key % static_cast<unsigned long long>(bp.n_s));
      const int s2 = static_cast<int>(sidx % w2) - cp.n[2];
      sidx /= w2;
      const int s1 = static_cast<int>(sidx % w1) - cp.n[1];
      const int s0 = static_cast<int>(sidx / w1) - cp.n[0];
      if (j < 0 || j >= n) continue;   // never taken: both passes keep the same pairs
      double rx, ry, rz;
      pair_test(pi, load_pos(pos, j), s0, s1, s2, cp, &rx, &ry, &rz);
      const int at = base + rank;
      sender[at] = j;
      receiver[at] = i;
      edge_vec[3 * at + 0] = static_cast<float>(rx);
      edge_vec[3 * at + 1] = static_cast<float>(ry);
      edge_vec[3 * at + 2] = static_cast<float>(rz);
      if (shift) {
        shift[3 * at + 0] = s0;
        shift[3 * at + 1] = s1;
        shift[3 * at + 2] = s2;
      }
    }
  }
}

// Nearest-image lists are symmetric with at most one image per pair, and the image of j <- i is
// minus that of i <- j (rint and the clamp are odd functions). So the transposed order needs no
// sort: the edges j sends, in receiver order, are the reverses of row j's edges in sender order,
// t_row_ptr = row_ptr and t_perm[m] = id of the reverse of edge m (sender j found in row i).
__global__ void k_reverse_edges(const int* __restrict__ row_ptr, const int* __restrict__ sender,
                                const int* __restrict__ receiver, int n_edges, int* __restrict__ t_perm) {
  for (int m = blockIdx.x * blockDim.x + threadIdx.x; m < n_edges; m += gridDim.x * blockDim.x) {
    const int j = receiver[m];
    const int i = sender[m];
    int lo = row_ptr[i], hi = row_ptr[i + 1];   // first entry of row i with sender >= j
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (sender[mid] < j) lo = mid + 1; else hi = mid;
    }
    t_perm[m] = lo;
  }
}

__global__ void k_iota(int* __restrict__ v, int n) {
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < n; k += gridDim.x * blockDim.x) v[k] = k;
}

// ptr[r] = first k with keys[k] >= r (keys sorted), r = 0..n_nodes: every entry is written once,
// by the edge at which the key passes r (or by the last edge / thread 0 at the ends).
__global__ void k_ptr_from_sorted(const int* __restrict__ keys, int n_keys, int n_nodes, int* __restrict__ ptr) {
  if (n_keys == 0) {
    for (int r = blockIdx.x * blockDim.x + threadIdx.x; r <= n_nodes; r += gridDim.x * blockDim.x) ptr[r] = 0;
    return;
  }
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k <= n_keys; k += gridDim.x * blockDim.x) {
    const int lo = k == 0 ? 0 : keys[k - 1] + 1;      // keys in (keys[k-1], keys[k]] start at k
    const int hi = k == n_keys ? n_nodes : keys[k];
    for (int r = lo; r <= hi; ++r) ptr[r] = k;
  }
}

__global__ void k_gather_key(const int* __restrict__ key_src, const int* __restrict__ idx, int n,
                             int* __restrict__ out) {
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < n; k += gridDim.x * blockDim.x) out[k] = key_src[idx[k]];
}

__global__ void k_gather_edges(const int* __restrict__ perm, int n, const int* __restrict__ sender_in,
                               const float* __restrict__ vec_in, int* __restrict__ sender,
                               float* __restrict__ vec) {
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < n; k += gridDim.x * blockDim.x) {
    const int e = perm[k];
    sender[k] = sender_in[e];
    vec[3 * k + 0] = vec_in[3 * e + 0];
    vec[3 * k + 1] = vec_in[3 * e + 1];
    vec[3 * k + 2] = vec_in[3 * e + 2];
  }
}

__global__ void k_check_range(const int* __restrict__ a, const int* __restrict__ b, int n, int n_nodes,
                              int* __restrict__ flag) {
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < n; k += gridDim.x * blockDim.x) {
    if (a[k] < 0 || a[k] >= n_nodes || b[k] < 0 || b[k] >= n_nodes) atomicOr(flag, 1);
  }
}

int key_bits(int n_nodes) {
  int b = 1;
  while ((1LL << b) <= n_nodes) ++b;
  return b;
}

int n_chunks_of(int n_nodes) { return n_nodes > 0 ? (n_nodes + kChunk - 1) / kChunk : 1; }

struct GraphWs {
  int* counts;   // n_nodes * n_chunks (+1)
  int* incl;     // n_nodes * n_chunks
  int* ka;
  int* kb;
  int* va;
  int* vb;
  int* pm;
  int* flag;
  // binned search: per-atom bin keys (sorted and in atom order), atom ids, wrap counts
  unsigned long long* bkey;
  unsigned long long* bkey_sorted;
  int* batom;
  int* batom_sorted;
  int* wrap;
  void* cub_tmp;
  size_t cub_bytes;
};

size_t cub_temp_bytes(int n_nodes, int max_edges) {
  size_t scan_b = 0, sort_b = 0;
  const long long n_cnt = static_cast<long long>(n_nodes > 0 ? n_nodes : 1) * n_chunks_of(n_nodes);
  cub::DeviceScan::InclusiveSum(nullptr, scan_b, static_cast<const int*>(nullptr),
                                static_cast<int*>(nullptr), static_cast<int>(n_cnt));
  cub::DeviceRadixSort::SortPairs(nullptr, sort_b, static_cast<const int*>(nullptr),
                                  static_cast<int*>(nullptr), static_cast<const int*>(nullptr),
                                  static_cast<int*>(nullptr), max_edges > 0 ? max_edges : 1, 0,
                                  key_bits(n_nodes));
  size_t bin_b = 0;
  cub::DeviceRadixSort::SortPairs(nullptr, bin_b, static_cast<const unsigned long long*>(nullptr),
                                  static_cast<unsigned long long*>(nullptr), static_cast<const int*>(nullptr),
                                  static_cast<int*>(nullptr), n_nodes > 0 ? n_nodes : 1, 0, 63);
  const size_t m = scan_b > sort_b ? scan_b : sort_b;
  return m > bin_b ? m : bin_b;
}

// bytes of the binned search's per-atom arrays
size_t bin_bytes(int n_nodes) {
  const size_t n = static_cast<size_t>(n_nodes > 0 ? n_nodes : 1);
  return 2 * align256(8 * n) + 2 * align256(4 * n) + align256(12 * n);
}

GraphWs carve(void* ws, int n_nodes, int max_edges) {
  char* p = static_cast<char*>(ws);
  GraphWs g;
  const size_t eb = align256(sizeof(int) * static_cast<size_t>(max_edges > 0 ? max_edges : 1));
  const size_t cb = align256(sizeof(int) * (static_cast<size_t>(n_nodes) * n_chunks_of(n_nodes) + 1));
  g.counts = reinterpret_cast<int*>(p);
  p += cb;
  g.incl = reinterpret_cast<int*>(p);
  p += cb;
  g.ka = reinterpret_cast<int*>(p); p += eb;
  g.kb = reinterpret_cast<int*>(p); p += eb;
  g.va = reinterpret_cast<int*>(p); p += eb;
  g.vb = reinterpret_cast<int*>(p); p += eb;
  g.pm = reinterpret_cast<int*>(p); p += eb;
  g.flag = reinterpret_cast<int*>(p); p += 256;
  const size_t n = static_cast<size_t>(n_nodes > 0 ? n_nodes : 1);
  g.bkey = reinterpret_cast<unsigned long long*>(p); p += align256(8 * n);
  g.bkey_sorted = reinterpret_cast<unsigned long long*>(p); p += align256(8 * n);
  g.batom = reinterpret_cast<int*>(p); p += align256(4 * n);
  g.batom_sorted = reinterpret_cast<int*>(p); p += align256(4 * n);
  g.wrap = reinterpret_cast<int*>(p); p += align256(12 * n);
  g.cub_tmp = p;
  g.cub_bytes = cub_temp_bytes(n_nodes, max_edges);
  return g;
}

int grid_for(long long n, int threads) {
  long long b = (n + threads - 1) / threads;
  if (b < 1) b = 1;
  if (b > 148 * 32) b = 148 * 32;
  return static_cast<int>(b);
}

// t_perm = stable sort of canonical edge ids by sender; t_row_ptr from the sorted keys.
etp_status transpose(int n_nodes, int n_edges, const int* sender, int* t_row_ptr, int* t_perm,
                     GraphWs& g, cudaStream_t s) {
  if (n_edges > 0) {
    k_iota<<<grid_for(n_edges, 256), 256, 0, s>>>(g.va, n_edges);
    size_t tb = g.cub_bytes;
    cudaError_t e = cub::DeviceRadixSort::SortPairs(g.cub_tmp, tb, sender, g.kb, g.va, t_perm, n_edges,
                                                    0, key_bits(n_nodes), s);
    if (e != cudaSuccess) return cuda_status(e, "transpose sort");
  }
  k_ptr_from_sorted<<<grid_for((n_edges > n_nodes ? n_edges : n_nodes) + 1, 256), 256, 0, s>>>(g.kb, n_edges,
                                                                                          n_nodes, t_row_ptr);
  return cuda_status(cudaGetLastError(), "transpose");
}


enum class NbrMode { kAuto, kAllPairs, kBins };

// ETP_NEIGHBORS = "bins" or "all-pairs" forces a search; unset, empty or "default" chooses.
NbrMode nbr_mode() {
  const char* v = std::getenv("ETP_NEIGHBORS");
  if (!v || !*v) return NbrMode::kAuto;
  const std::string m(v);
  if (m == "bins") return NbrMode::kBins;
  if (m == "all-pairs") return NbrMode::kAllPairs;
  return NbrMode::kAuto;
}

// The bin layout (see BinParams). Returns whether binning is worth it by default: at least 2048
// atoms, and on a fully periodic cell at least 4 x 4 x 4 bins (with fewer, every receiver scans
// nearly every atom anyway). bp->n_off = 0 when no layout can be built.
bool plan_bins(const double* cell, const int* pbc, double rc, int n_nodes, const CellParams& cp, BinParams* bp) {
  bp->n_off = 0;
  bp->n_s = static_cast<long long>(2 * cp.n[0] + 1) * (2 * cp.n[1] + 1) * (2 * cp.n[2] + 1);
  if (!(rc > 0.0) || !std::isfinite(rc)) return false;
  const double rcm = rc * (1.0 + 1e-6);
  double spacing[3] = {1.0, 1.0, 1.0};
  for (int k = 0; k < 9; ++k) bp->inv[k] = (k % 4 == 0) ? 1.0 : 0.0;
  if (cell) {
    const double* c = cell;
    const double det = c[0] * (c[4] * c[8] - c[5] * c[7]) - c[1] * (c[3] * c[8] - c[5] * c[6]) +
                       c[2] * (c[3] * c[7] - c[4] * c[6]);
    if (!(std::fabs(det) > 0.0)) return false;
    // inverse by cofactors: inv[3 k + a] = cof(a, k) / det
    bp->inv[0] = (c[4] * c[8] - c[5] * c[7]) / det;
    bp->inv[1] = (c[2] * c[7] - c[1] * c[8]) / det;
    bp->inv[2] = (c[1] * c[5] - c[2] * c[4]) / det;
    bp->inv[3] = (c[5] * c[6] - c[3] * c[8]) / det;
    bp->inv[4] = (c[0] * c[8] - c[2] * c[6]) / det;
    bp->inv[5] = (c[2] * c[3] - c[0] * c[5]) / det;
    bp->inv[6] = (c[3] * c[7] - c[4] * c[6]) / det;
    bp->inv[7] = (c[1] * c[6] - c[0] * c[7]) / det;
    bp->inv[8] = (c[0] * c[4] - c[1] * c[3]) / det;
    for (int a = 0; a < 3; ++a) {
      const double* u = c + 3 * ((a + 1) % 3);
      const double* w = c + 3 * ((a + 2) % 3);
      const double cx = u[1] * w[2] - u[2] * w[1], cy = u[2] * w[0] - u[0] * w[2], cz = u[0] * w[1] - u[1] * w[0];
      spacing[a] = std::fabs(det) / std::sqrt(cx * cx + cy * cy + cz * cz);
      if (!(spacing[a] > 0.0)) return false;
    }
  }
  long long periodic_bins = 1;
  bool all_periodic = true;
  bp->n_off = 1;
  for (int a = 0; a < 3; ++a) {
    bp->periodic[a] = (cell && pbc && pbc[a]) ? 1 : 0;
    if (bp->periodic[a]) {
      const double per = std::floor(spacing[a] / rcm);
      bp->nb[a] = per >= 1.0 ? (per < 1e6 ? static_cast<int>(per) : 1000000) : 1;
      bp->K[a] = static_cast<int>(std::ceil(rcm * bp->nb[a] / spacing[a]));
      if (bp->K[a] < 1) bp->K[a] = 1;
      bp->width[a] = 1.0 / bp->nb[a];
      periodic_bins *= bp->nb[a];
    } else {
      all_periodic = false;
      bp->nb[a] = 1;
      bp->K[a] = 1;
      bp->width[a] = rcm / spacing[a];
    }
    if (bp->K[a] > 8) {   // a cell far thinner than r_cut: nothing to gain from bins
      bp->n_off = 0;
      return false;
    }
    bp->n_off *= 2 * bp->K[a] + 1;
  }
  if (n_nodes < 2048) return false;
  return !(all_periodic && periodic_bins < 64);
}

// All-pairs search: row_ptr, sender, edge_vec, shift and the receiver of every edge (g.ka).
etp_status neighbors_all_pairs(const float* pos, int n_nodes, const CellParams& cp, int max_edges, int* n_edges,
                               int* row_ptr, int* sender, float* edge_vec, int* shift, GraphWs& g, cudaStream_t s) {
  cudaError_t e;
  const int n_chunks = n_chunks_of(n_nodes);
  const long long n_tasks = static_cast<long long>(n_nodes) * n_chunks;
  const int task_blocks = grid_for(n_tasks * 32, 256);
  if (n_nodes > 0) {
    k_nbr_count<<<task_blocks, 256, 0, s>>>(pos, n_nodes, n_chunks, cp, g.counts);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e, "neighbour count");
    size_t tb = g.cub_bytes;
    e = cub::DeviceScan::InclusiveSum(g.cub_tmp, tb, g.counts, g.incl, static_cast<int>(n_tasks), s);
    if (e != cudaSuccess) return cuda_status(e, "neighbour scan");
  }
  k_row_ptr_chunks<<<grid_for(n_nodes + 1, 256), 256, 0, s>>>(g.incl, n_nodes, n_chunks, row_ptr);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e, "row pointers");
  int total = 0;
  if ((e = cudaMemcpyAsync(&total, row_ptr + n_nodes, sizeof(int), cudaMemcpyDeviceToHost, s)) != cudaSuccess)
    return cuda_status(e, "read edge count");
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return cuda_status(e, "neighbour count sync");
  *n_edges = total;
  if (total > max_edges) {
    set_error("etp_neighbors: " + std::to_string(total) + " edges exceed max_edges");
    return ETP_ERR_CAPACITY;
  }
  if (n_nodes > 0 && total > 0) {
    k_nbr_emit<<<task_blocks, 256, 0, s>>>(pos, n_nodes, n_chunks, cp, g.counts, g.incl, sender, edge_vec, shift,
                                           g.ka);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e, "neighbour emit");
  }
  return ETP_OK;
}

// Binned search, same outputs. *done = false (nothing written that the all-pairs search does not
// rewrite) when a coordinate falls outside the representable bin range.
etp_status neighbors_binned(const float* pos, int n_nodes, const CellParams& cp, const BinParams& bp, int max_edges,
                            int* n_edges, int* row_ptr, int* sender, float* edge_vec, int* shift, GraphWs& g,
                            cudaStream_t s, bool* done) {
  *done = false;
  cudaError_t e;
  if ((e = cudaMemsetAsync(g.flag, 0, sizeof(int), s)) != cudaSuccess) return cuda_status(e, "memset");
  k_bin_atoms<<<grid_for(n_nodes, 256), 256, 0, s>>>(pos, n_nodes, bp, g.bkey, g.batom, g.wrap, g.flag);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e, "bin atoms");
  size_t tb = g.cub_bytes;
  e = cub::DeviceRadixSort::SortPairs(g.cub_tmp, tb, g.bkey, g.bkey_sorted, g.batom, g.batom_sorted, n_nodes, 0, 63,
                                      s);
  if (e != cudaSuccess) return cuda_status(e, "bin sort");
  const int warp_blocks = grid_for(static_cast<long long>(n_nodes) * 32, 256);
  k_bin_pairs<false><<<warp_blocks, 256, 0, s>>>(pos, n_nodes, cp, bp, g.bkey_sorted, g.batom_sorted, g.bkey, g.wrap,
                                                 g.counts, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e, "binned count");
  tb = g.cub_bytes;
  e = cub::DeviceScan::InclusiveSum(g.cub_tmp, tb, g.counts, g.incl, n_nodes, s);
  if (e != cudaSuccess) return cuda_status(e, "binned scan");
  k_row_ptr_chunks<<<grid_for(n_nodes + 1, 256), 256, 0, s>>>(g.incl, n_nodes, 1, row_ptr);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e, "row pointers");
  int total = 0, flag = 0;
  if ((e = cudaMemcpyAsync(&total, row_ptr + n_nodes, sizeof(int), cudaMemcpyDeviceToHost, s)) != cudaSuccess)
    return cuda_status(e, "read edge count");
  if ((e = cudaMemcpyAsync(&flag, g.flag, sizeof(int), cudaMemcpyDeviceToHost, s)) != cudaSuccess)
    return cuda_status(e, "read bin flag");
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return cuda_status(e, "neighbour count sync");
  if (flag) return ETP_OK;   // coordinates beyond the bin range: the caller scans all pairs
  *done = true;
  *n_edges = total;
  if (total > max_edges) {
    set_error("etp_neighbors: " + std::to_string(total) + " edges exceed max_edges");
    return ETP_ERR_CAPACITY;
  }
  if (total == 0) return ETP_OK;
  // the rows' edge keys (sender * n_s + image index), in bin order, in [kb, va)
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(g.kb);
  k_bin_pairs<true><<<warp_blocks, 256, 0, s>>>(pos, n_nodes, cp, bp, g.bkey_sorted, g.batom_sorted, g.bkey, g.wrap,
                                                nullptr, row_ptr, keys, g.ka, sender, edge_vec, shift);
  return cuda_status(cudaGetLastError(), "binned emit");
}

}  // namespace

size_t graph_workspace_bytes(int n_nodes, int max_edges) {
  const size_t eb = align256(sizeof(int) * static_cast<size_t>(max_edges > 0 ? max_edges : 1));
  const size_t cb = align256(sizeof(int) * (static_cast<size_t>(n_nodes) * n_chunks_of(n_nodes) + 1));
  return 2 * cb + 5 * eb + 256 + bin_bytes(n_nodes) + align256(cub_temp_bytes(n_nodes, max_edges));
}

etp_status neighbors(const float* pos, int n_nodes, const double* cell, const int* pbc,
                     float r_cut, int max_edges, int* n_edges, int* row_ptr, int* sender,
                     float* edge_vec, int* shift, int* t_row_ptr, int* t_perm, void* ws,
                     size_t ws_bytes, cudaStream_t s) {
  (void)ws_bytes;
  CellParams cp;
  for (int k = 0; k < 9; ++k) cp.c[k] = cell ? cell[k] : 0.0;
  const double rc = static_cast<double>(r_cut);
  cp.rc2 = rc * rc;
  if (cell) {
    const double* c = cell;
    const double vol = std::fabs(c[0] * (c[4] * c[8] - c[5] * c[7]) - c[1] * (c[3] * c[8] - c[5] * c[6]) +
                                 c[2] * (c[3] * c[7] - c[4] * c[6]));
    for (int a = 0; a < 3; ++a) {
      cp.n[a] = 0;
      if (!pbc || !pbc[a]) continue;
      const double* b = c + 3 * ((a + 1) % 3);
      const double* d = c + 3 * ((a + 2) % 3);
      const double cx = b[1] * d[2] - b[2] * d[1], cy = b[2] * d[0] - b[0] * d[2], cz = b[0] * d[1] - b[1] * d[0];
      const double spacing = vol / std::sqrt(cx * cx + cy * cy + cz * cz);
      if (!(spacing > 0.0)) {
        set_error("etp_neighbors: degenerate cell");
        return ETP_ERR_INVALID_ARG;
      }
      cp.n[a] = static_cast<int>(std::ceil(rc / spacing));
    }
    const bool ortho = c[1] == 0.0 && c[2] == 0.0 && c[3] == 0.0 && c[5] == 0.0 && c[6] == 0.0 && c[7] == 0.0;
    cp.min_image = ortho ? 1 : 0;
    for (int a = 0; a < 3; ++a) {
      cp.len[a] = c[4 * a];   // signed: the image shift along axis a is S_a * c[a][a]
      if (cp.n[a] > 0 && !(std::fabs(cp.len[a]) > 2.0 * rc)) cp.min_image = 0;
    }
  } else {
    cp.min_image = 0;
    cp.len[0] = cp.len[1] = cp.len[2] = 0.0;
    if (pbc && (pbc[0] || pbc[1] || pbc[2])) {
      set_error("etp_neighbors: periodic axes need a cell");
      return ETP_ERR_INVALID_ARG;
    }
    cp.n[0] = cp.n[1] = cp.n[2] = 0;
  }
  GraphWs g = carve(ws, n_nodes, max_edges);
  BinParams bp;
  const NbrMode mode = nbr_mode();
  const bool bins_help = plan_bins(cell, pbc, rc, n_nodes, cp, &bp);
  const bool use_bins = n_nodes > 0 && cp.rc2 > 0.0 && mode != NbrMode::kAllPairs &&
                        (mode == NbrMode::kBins ? bp.n_off > 0 : bins_help);
  etp_status st = ETP_OK;
  bool done = false;
  if (use_bins) {
    st = neighbors_binned(pos, n_nodes, cp, bp, max_edges, n_edges, row_ptr, sender, edge_vec, shift, g, s, &done);
    if (st != ETP_OK) return st;
  }
  if (!done) {
    st = neighbors_all_pairs(pos, n_nodes, cp, max_edges, n_edges, row_ptr, sender, edge_vec, shift, g, s);
    if (st != ETP_OK) return st;
  }
  const int total = *n_edges;
  cudaError_t e;
  if (cp.min_image) {
    e = cudaMemcpyAsync(t_row_ptr, row_ptr, sizeof(int) * (static_cast<size_t>(n_nodes) + 1),
                        cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_status(e, "transposed row pointers");
    if (total > 0) k_reverse_edges<<<grid_for(total, 256), 256, 0, s>>>(row_ptr, sender, g.ka, total, t_perm);
    return cuda_status(cudaGetLastError(), "reverse edges");
  }
  return transpose(n_nodes, total, sender, t_row_ptr, t_perm, g, s);
}

etp_status build_csr(int n_nodes, int n_edges, const int* receiver, const int* sender_in,
                     const float* edge_vec_in, int* row_ptr, int* sender, float* edge_vec,
                     int* perm, int* t_row_ptr, int* t_perm, void* ws, size_t ws_bytes,
                     cudaStream_t s) {
  (void)ws_bytes;
  GraphWs g = carve(ws, n_nodes, n_edges);
  cudaError_t e;
  int* pm = perm ? perm : g.pm;
  if (n_edges > 0) {
    if ((e = cudaMemsetAsync(g.flag, 0, sizeof(int), s)) != cudaSuccess) return cuda_status(e, "memset");
    k_check_range<<<grid_for(n_edges, 256), 256, 0, s>>>(receiver, sender_in, n_edges, n_nodes, g.flag);
    int bad = 0;
    if ((e = cudaMemcpyAsync(&bad, g.flag, sizeof(int), cudaMemcpyDeviceToHost, s)) != cudaSuccess)
      return cuda_status(e, "read flag");
    if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return cuda_status(e, "build_csr sync");
    if (bad) {
      set_error("etp_build_csr: receiver or sender index out of [0, n_nodes)");
      return ETP_ERR_BAD_GRAPH;
    }
    const int bits = key_bits(n_nodes);
    k_iota<<<grid_for(n_edges, 256), 256, 0, s>>>(g.va, n_edges);
    size_t tb = g.cub_bytes;
    // LSD: stable by sender, then stable by receiver -> (receiver, sender, input index)
    e = cub::DeviceRadixSort::SortPairs(g.cub_tmp, tb, sender_in, g.kb, g.va, g.vb, n_edges, 0, bits, s);
    if (e != cudaSuccess) return cuda_status(e, "csr sort 1");
    k_gather_key<<<grid_for(n_edges, 256), 256, 0, s>>>(receiver, g.vb, n_edges, g.ka);
    tb = g.cub_bytes;
    e = cub::DeviceRadixSort::SortPairs(g.cub_tmp, tb, g.ka, g.kb, g.vb, pm, n_edges, 0, bits, s);
    if (e != cudaSuccess) return cuda_status(e, "csr sort 2");
    k_gather_edges<<<grid_for(n_edges, 256), 256, 0, s>>>(pm, n_edges, sender_in, edge_vec_in, sender, edge_vec);
  }
  k_ptr_from_sorted<<<grid_for((n_edges > n_nodes ? n_edges : n_nodes) + 1, 256), 256, 0, s>>>(g.kb, n_edges,
                                                                                          n_nodes, row_ptr);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e, "build_csr");
  return transpose(n_nodes, n_edges, sender, t_row_ptr, t_perm, g, s);
}

}  // namespace etp
