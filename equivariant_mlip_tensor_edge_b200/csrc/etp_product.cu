// Node-local product ladder (the second workload of the pages: FlashCart Fig. 3b / Fig. E1):
//
//   B_1 = A,   B_{q+1}[l3, m3, u] = sum_{p = (l1, l2, l3)} W_q[p, u] sum_{m1, m2} C B_q[l1, m1, u] A[l2, m2, u],
//   out = sum_{q = 1..nu} B_q,
//
// the path-reduced "uvu" product with a scalar weight per path and channel, the same path set as the
// edge convolution. Every node and channel is independent, so a thread holds K channels of one node
// (lanes along the channels: each component row is one coalesced access per warp) and runs the whole
// ladder in registers: A is read once and out written once, whatever nu.
#include <cstdint>
#include <string>

#include "etp_device.h"
#include "etp_internal.h"

namespace etp {
namespace {

// Channels per thread: 2 (one 8-byte access per component row; measured faster than 1 or 4 at
// 4096 nodes x 128 channels for every rank and order 2..5 but one, where it is within 5%).
constexpr int kNodeK = 2;

#define ETP_NODE_BIND(LL)                                                                              \
  template <int K, class WF>                                                                           \
  __device__ __forceinline__ void tp_node(IntLN<LL>, const float (&b)[Gen<LL>::D][K],                  \
                                          const float (&a)[Gen<LL>::D][K], WF&& wf,                    \
                                          float (&acc)[Gen<LL>::D][K]) {                               \
    etp_gen::tp_node_##LL<K>(b, a, wf, acc);                                                          \
  }
template <int L> struct IntLN {};
ETP_NODE_BIND(1)
ETP_NODE_BIND(2)
ETP_NODE_BIND(3)
#undef ETP_NODE_BIND

template <int K>
__device__ __forceinline__ void load_k(const float* p, float (&v)[K]) {
  if constexpr (K == 4) {
    const float4 t = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
  } else {
    const float2 t = __ldg(reinterpret_cast<const float2*>(p));
    v[0] = t.x; v[1] = t.y;
  }
}

template <int K>
__device__ __forceinline__ void store_k(float* p, const float (&v)[K]) {
  if constexpr (K == 4) *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  else *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
}

template <int D, int K>
__device__ __forceinline__ void load_item(const float* A, int C, int node, int ch, float (&v)[D][K]) {
  const float* ar = A + static_cast<size_t>(node) * D * C + ch;
#pragma unroll
  for (int c = 0; c < D; ++c) load_k<K>(ar + c * C, v[c]);
}

// W: [nu - 1][P][C]
template <int L>
__global__ void __launch_bounds__(256) k_node_ladder(int n_nodes, int C, int nu, const float* __restrict__ A,
                                                     const float* __restrict__ W, float* __restrict__ out) {
  constexpr int D = Gen<L>::D, P = Gen<L>::P, K = kNodeK;
  const int groups = C / K;
  // item t = node * groups + channel group; the grid-stride walk advances (node, group) by the
  // stride's quotient and remainder instead of dividing every item (the launch keeps
  // n_nodes * groups below 2^31)
  const int stride = gridDim.x * blockDim.x;
  const int d_node = stride / groups, d_grp = stride - d_node * groups;
  const int t0 = blockIdx.x * blockDim.x + threadIdx.x;
  int node = t0 / groups, grp = t0 - node * groups;
  // the grid holds only what is resident, so a thread takes several (node, channel-pair) items: the
  // next item's rows are requested before the current item's products, which hides their latency
  float an[D][K];
  if (node < n_nodes) load_item<D, K>(A, C, node, grp * K, an);
  while (node < n_nodes) {
    const int ch = grp * K;
    int next_node = node + d_node, next_grp = grp + d_grp;
    if (next_grp >= groups) {
      next_grp -= groups;
      ++next_node;
    }
    float a[D][K], b[D][K], o[D][K];
#pragma unroll
    for (int c = 0; c < D; ++c)
#pragma unroll
      for (int k = 0; k < K; ++k) {
        a[c][k] = an[c][k];
        b[c][k] = an[c][k];
        o[c][k] = an[c][k];
      }
    if (next_node < n_nodes) load_item<D, K>(A, C, next_node, next_grp * K, an);
    for (int q = 0; q + 1 < nu; ++q) {
      const float* wq = W + static_cast<size_t>(q) * P * C + ch;
      float acc[D][K];
#pragma unroll
      for (int c = 0; c < D; ++c)
#pragma unroll
        for (int k = 0; k < K; ++k) acc[c][k] = 0.0f;
      // (array bound spelled kNodeK: a generic lambda whose parameter is sized by a local constexpr
      // of the kernel template crashes the CUDA 12.9 front end)
      tp_node(IntLN<L>{}, b, a, [&](auto pc, float (&wp)[kNodeK]) {
        constexpr int p = decltype(pc)::value;
        load_k<kNodeK>(wq + p * C, wp);
      }, acc);
#pragma unroll
      for (int c = 0; c < D; ++c)
#pragma unroll
        for (int k = 0; k < K; ++k) {
          b[c][k] = acc[c][k];
          o[c][k] += acc[c][k];
        }
    }
    float* orow = out + static_cast<size_t>(node) * D * C + ch;
#pragma unroll
    for (int c = 0; c < D; ++c) store_k<K>(orow + c * C, o[c]);
    node = next_node;
    grp = next_grp;
  }
}

int g_nsms = 0;
int nnum_sms() {
  if (g_nsms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_nsms, cudaDevAttrMultiProcessorCount, dev);
    if (g_nsms <= 0) g_nsms = 148;
  }
  return g_nsms;
}

template <int L>
etp_status ladder_launch(int channels, int n_nodes, int nu, const float* A, const float* W, float* out,
                         cudaStream_t s) {
  static int per_sm = 0;
  if (per_sm == 0) {
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_node_ladder<L>, 256, 0);
    if (per_sm <= 0) per_sm = 1;
  }
  const long long total = static_cast<long long>(n_nodes) * (channels / kNodeK);
  long long blocks = (total + 255) / 256;
  if (blocks > static_cast<long long>(per_sm) * nnum_sms()) blocks = static_cast<long long>(per_sm) * nnum_sms();
  if (blocks < 1) blocks = 1;
  k_node_ladder<L><<<static_cast<int>(blocks), 256, 0, s>>>(n_nodes, channels, nu, A, W, out);
  return cuda_status(cudaGetLastError(), "node ladder launch");
}

}  // namespace

etp_status launch_node_ladder(int lmax, int channels, int n_nodes, int nu, const float* A, const float* W,
                              float* out, cudaStream_t s) {
  switch (lmax) {
    case 1: return ladder_launch<1>(channels, n_nodes, nu, A, W, out, s);
    case 2: return ladder_launch<2>(channels, n_nodes, nu, A, W, out, s);
    case 3: return ladder_launch<3>(channels, n_nodes, nu, A, W, out, s);
  }
  set_error("etp_node_ladder: unsupported lmax");
  return ETP_ERR_UNSUPPORTED;
}

}  // namespace etp
