// Graph construction: brute-force neighbour list with a fixed float64 inclusion test, canonical
// receiver-sorted CSR, and the transposed (sender-sorted) order. Integer outputs are
// deterministic and bit-exact against any implementation of the same test (include/etp.h).
#include <cub/cub.cuh>

#include <cmath>
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
  return scan_b > sort_b ? scan_b : sort_b;
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

}  // namespace

size_t graph_workspace_bytes(int n_nodes, int max_edges) {
  const size_t eb = align256(sizeof(int) * static_cast<size_t>(max_edges > 0 ? max_edges : 1));
  const size_t cb = align256(sizeof(int) * (static_cast<size_t>(n_nodes) * n_chunks_of(n_nodes) + 1));
  return 2 * cb + 5 * eb + 256 + align256(cub_temp_bytes(n_nodes, max_edges));
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
