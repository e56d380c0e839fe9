// C ABI of libetp: handle lifecycle, argument checks, workspace carving and kernel dispatch.
// The operation and conventions are documented in include/etp.h.
#include <cctype>
#include <cstdlib>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "etp_internal.h"
#include "generated/etp_paths.h"

struct etp_ctx {
  etp::Ctx c;
};

namespace {

// Gives the handle its sticky status word: pinned host memory mapped into the device address space
// where a device is present (the kernels store their timeout codes there), plain host memory
// otherwise (no kernel can run then). Returns false on failure (message set).
bool attach_status_word(etp_ctx* h) {
  int ndev = 0;
  cudaError_t e = cudaGetDeviceCount(&ndev);
  if (e == cudaSuccess && ndev > 0) {
    void* p = nullptr;
    e = cudaHostAlloc(&p, 64, cudaHostAllocMapped | cudaHostAllocPortable);
    void* d = nullptr;
    if (e == cudaSuccess) e = cudaHostGetDevicePointer(&d, p, 0);
    if (e != cudaSuccess) {
      if (p) cudaFreeHost(p);
      etp::cuda_status(e, "etp_create: pinned status word");
      return false;
    }
    *static_cast<volatile int*>(p) = 0;
    h->c.status = static_cast<int*>(p);
    h->c.status_dev = static_cast<int*>(d);
    h->c.status_mapped = true;
    return true;
  }
  cudaGetLastError();   // no device: clear the runtime's error state
  void* p = std::calloc(1, 64);
  if (!p) {
    etp::set_error("etp_create: out of host memory");
    return false;
  }
  h->c.status = static_cast<int*>(p);
  h->c.status_dev = nullptr;
  h->c.status_mapped = false;
  return true;
}

void release_status_word(etp_ctx* h) {
  if (!h || !h->c.status) return;
  if (h->c.status_mapped) cudaFreeHost(h->c.status);
  else std::free(h->c.status);
  h->c.status = nullptr;
}

}  // namespace

namespace etp {

static thread_local std::string g_last_error;

void set_error(const std::string& msg) { g_last_error = msg; }

const Ctx* ctx_of(etp_handle h) { return h ? &h->c : nullptr; }

etp_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return ETP_OK;
  set_error(std::string(what) + ": " + cudaGetErrorString(e));
  return ETP_ERR_CUDA;
}

etp_status read_status(const Ctx& c, cudaStream_t s, const char* who) {
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_status(e, who);
  const int code = c.status ? *reinterpret_cast<volatile int*>(c.status) : 0;
  if (code != 0) {
    set_error(std::string(who) + ": a bounded pipeline wait gave up (code " + std::to_string(code) +
              "); the output is incomplete");
    return ETP_ERR_CUDA;
  }
  return ETP_OK;
}

// Entry gate of every compute call: a code left in the handle's status word by an earlier call's
// kernel fails the call until etp_get_status has read and cleared it.
static etp_status status_gate(const Ctx& c, const char* who) {
  const int code = c.status ? *reinterpret_cast<volatile int*>(c.status) : 0;
  if (code == 0) return ETP_OK;
  set_error(std::string(who) + ": a kernel of an earlier call on this handle gave up a bounded pipeline wait (code " +
            std::to_string(code) + "); outputs since then may be incomplete; etp_get_status reads and clears it");
  return ETP_ERR_CUDA;
}

etp_status gate(etp_handle h, const char* who) { return h ? status_gate(h->c, who) : ETP_OK; }

namespace {

struct Block {
  int mul, l, parity;
};

// "64x0e+64x1o" -> blocks. Returns false on a malformed string.
bool parse_irreps(const char* s, std::vector<Block>* out) {
  if (!s) return false;
  std::string str;
  for (const char* p = s; *p; ++p)
    if (!std::isspace(static_cast<unsigned char>(*p))) str.push_back(*p);
  if (str.empty()) return false;
  size_t pos = 0;
  while (pos <= str.size()) {
    size_t end = str.find('+', pos);
    if (end == std::string::npos) end = str.size();
    std::string term = str.substr(pos, end - pos);
    if (term.empty()) return false;
    int mul = 1;
    size_t x = term.find('x');
    std::string lp = term;
    if (x != std::string::npos) {
      std::string m = term.substr(0, x);
      if (m.empty() || m.size() > 6) return false;
      for (char ch : m)
        if (!std::isdigit(static_cast<unsigned char>(ch))) return false;
      mul = std::atoi(m.c_str());
      lp = term.substr(x + 1);
    }
    if (lp.size() < 2 || lp.size() > 3) return false;
    char par = lp.back();
    if (par != 'e' && par != 'o') return false;
    std::string ls = lp.substr(0, lp.size() - 1);
    for (char ch : ls)
      if (!std::isdigit(static_cast<unsigned char>(ch))) return false;
    out->push_back({mul, std::atoi(ls.c_str()), par == 'e' ? 1 : -1});
    pos = end + 1;
    if (end == str.size()) break;
  }
  return true;
}

// Paths (block_in, l2, block_out) in lexicographic order with the triangle and parity rules.
std::vector<int> enumerate_paths(const std::vector<Block>& in, int sh_lmax, const std::vector<Block>& out) {
  std::vector<int> ls;
  for (const Block& a : in)
    for (int l2 = 0; l2 <= sh_lmax; ++l2)
      for (const Block& b : out) {
        int sh_par = (l2 % 2) ? -1 : 1;
        if (std::abs(a.l - l2) <= b.l && b.l <= a.l + l2 && a.parity * sh_par == b.parity) {
          ls.push_back(a.l);
          ls.push_back(l2);
          ls.push_back(b.l);
        }
      }
  return ls;
}

template <int L>
bool fill_from_table(Ctx* c, const std::vector<int>& ls) {
  using PS = etp_gen::PathSet<L>;
  const int* tab = L == 1 ? etp_gen::kPathL_1 : (L == 2 ? etp_gen::kPathL_2 : etp_gen::kPathL_3);
  if (static_cast<int>(ls.size()) != 3 * PS::P) return false;
  for (int i = 0; i < 3 * PS::P; ++i)
    if (ls[i] != tab[i]) return false;
  c->n_paths = PS::P;
  c->cg_nnz = PS::NNZ;
  c->sum_2l3p1 = PS::SUM_2L3P1;
  return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The uniform kernels' configuration: C x (0e + 1o + ... + Le) in and out, sh_lmax = L, 1 <= L <= 3,
// C a multiple of 4 in [4, 256].
bool uniform_config(const std::vector<Block>& bin, int sh_lmax, const std::vector<Block>& bout) {
  const int L = static_cast<int>(bin.size()) - 1;
  if (L < 1 || L > kMaxL || bin.size() != bout.size() || sh_lmax != L) return false;
  const int C = bin[0].mul;
  for (int l = 0; l <= L; ++l) {
    const int par = (l % 2) ? -1 : 1;
    const Block& a = bin[l];
    const Block& b = bout[l];
    if (a.l != l || b.l != l || a.parity != par || b.parity != par || a.mul != C || b.mul != C) return false;
  }
  return C % kBatch == 0 && C >= kBatch && C <= 256;
}

// General irreps: paths (block_in, l2, block_out), lexicographic, with the triangle rule, parity
// p1 (-1)^l2 = p3 and equal multiplicities (uvu pairs channel u with channel u).
bool general_config(const std::vector<Block>& bin, int sh_lmax, const std::vector<Block>& bout, float r_cut,
                    Ctx* c, std::string* why) {
  if (sh_lmax > etp_gen::kGenLmax) {
    *why = "sh_lmax above 4";
    return false;
  }
  if (bin.size() > static_cast<size_t>(kGenMaxBlocks) || bout.size() > static_cast<size_t>(kGenMaxBlocks)) {
    *why = "more than 16 blocks";
    return false;
  }
  GenParams& g = c->gen;
  int lmax = sh_lmax;
  std::vector<int> in_off, out_off;
  int off = 0;
  for (const Block& b : bin) {
    if (b.l > etp_gen::kGenLmax || b.mul < 1 || b.mul > 1024) {
      *why = "blocks need 0 <= l <= 4 and 1 <= multiplicity <= 1024";
      return false;
    }
    in_off.push_back(off);
    off += b.mul * (2 * b.l + 1);
    lmax = b.l > lmax ? b.l : lmax;
  }
  g.dim_in = off;
  off = 0;
  for (const Block& b : bout) {
    if (b.l > etp_gen::kGenLmax || b.mul < 1 || b.mul > 1024) {
      *why = "blocks need 0 <= l <= 4 and 1 <= multiplicity <= 1024";
      return false;
    }
    out_off.push_back(off);
    off += b.mul * (2 * b.l + 1);
    lmax = b.l > lmax ? b.l : lmax;
  }
  g.dim_out = off;
  if (g.dim_in > kGenMaxDim || g.dim_out > kGenMaxDim) {
    *why = "node rows longer than 4096 floats";
    return false;
  }
  int n = 0, cols = 0, nnz = 0, s3 = 0;
  for (size_t a = 0; a < bin.size(); ++a)
    for (int l2 = 0; l2 <= sh_lmax; ++l2)
      for (size_t b = 0; b < bout.size(); ++b) {
        const Block& A = bin[a];
        const Block& B = bout[b];
        const int sh_par = (l2 % 2) ? -1 : 1;
        if (!(std::abs(A.l - l2) <= B.l && B.l <= A.l + l2 && A.parity * sh_par == B.parity && A.mul == B.mul))
          continue;
        if (n == kGenMaxPaths) {
          *why = "more than 128 paths";
          return false;
        }
        const int tri = etp_gen::kGenTriId[(A.l * 5 + l2) * 5 + B.l];
        g.p[n] = GenPath{in_off[a], out_off[b], cols, A.mul, tri};
        c->path_blocks[n][0] = static_cast<short>(a);
        c->path_blocks[n][1] = static_cast<short>(l2);
        c->path_blocks[n][2] = static_cast<short>(b);
        cols += A.mul;
        nnz += etp_gen::kGenTriNnz[tri];
        s3 += 2 * B.l + 1;
        c->flop_fwd += 2 * (etp_gen::kGenTriNnz[tri] + 2 * B.l + 1) * A.mul;
        c->flop_bwd += 2 * (3 * etp_gen::kGenTriNnz[tri] + 2 * (2 * B.l + 1)) * A.mul;
        ++n;
      }
  if (n == 0) {
    *why = "no path couples the two irreps";
    return false;
  }
  g.n_paths = n;
  g.cols = cols;
  // work groups: the output blocks (forward) and input blocks (backward) that some path touches
  for (int side = 0; side < 2; ++side) {
    const std::vector<Block>& blocks = side ? bin : bout;
    const std::vector<int>& offs = side ? in_off : out_off;
    GenGroup* grp = side ? g.in_grp : g.out_grp;
    unsigned char* order = side ? g.order_in : g.order_out;
    int ng = 0, k = 0, mx = 0;
    for (size_t b = 0; b < blocks.size(); ++b) {
      const int beg = k;
      for (int q = 0; q < n; ++q)
        if ((side ? g.p[q].in_off : g.p[q].out_off) == offs[b]) order[k++] = static_cast<unsigned char>(q);
      if (k == beg) continue;
      const int size = blocks[b].mul * (2 * blocks[b].l + 1);
      grp[ng++] = GenGroup{offs[b], size, beg, k};
      mx = size > mx ? size : mx;
    }
    if (side) {
      g.n_in_groups = ng;
      g.max_in_size = mx;
    } else {
      g.n_out_groups = ng;
      g.max_out_size = mx;
    }
  }
  g.sh_lmax = sh_lmax;
  g.inv_rc = 1.0f / r_cut;
  plan_general_tc(g);
  int mul = bin[0].mul;
  for (const Block& b : bin) mul = b.mul == mul ? mul : 0;
  for (const Block& b : bout) mul = b.mul == mul ? mul : 0;
  c->general = true;
  c->lmax = lmax;
  c->channels = mul;
  c->dim = g.dim_in;
  c->n_paths = n;
  c->cg_nnz = nnz;
  c->sum_2l3p1 = s3;
  c->r_cut = r_cut;
  return true;
}

}  // namespace
}  // namespace etp

using namespace etp;

extern "C" {

const char* etp_status_string(etp_status s) {
  switch (s) {
    case ETP_OK: return "ok";
    case ETP_ERR_INVALID_ARG: return "invalid argument";
    case ETP_ERR_IRREPS: return "malformed irreps string";
    case ETP_ERR_UNSUPPORTED: return "unsupported configuration";
    case ETP_ERR_BAD_GRAPH: return "invalid CSR graph";
    case ETP_ERR_CUDA: return "CUDA error";
    case ETP_ERR_CAPACITY: return "output capacity exceeded";
  }
  return "unknown status";
}

const char* etp_last_error(void) { return g_last_error.c_str(); }

etp_status etp_create(const char* irreps_in, int sh_lmax, const char* irreps_out, int n_basis,
                      float r_cut, etp_handle* out) {
  if (!out) {
    set_error("etp_create: out is NULL");
    return ETP_ERR_INVALID_ARG;
  }
  *out = nullptr;
  std::vector<Block> bin, bout;
  if (!parse_irreps(irreps_in, &bin) || !parse_irreps(irreps_out, &bout)) {
    set_error("etp_create: malformed irreps string");
    return ETP_ERR_IRREPS;
  }
  if (!(r_cut > 0.f) || n_basis <= 0 || sh_lmax < 0) {
    set_error("etp_create: r_cut must be > 0, n_basis > 0, sh_lmax >= 0");
    return ETP_ERR_INVALID_ARG;
  }
  if (n_basis != kNumBasis) {
    set_error("etp_create: only n_basis == 8 is implemented");
    return ETP_ERR_UNSUPPORTED;
  }
  if (!uniform_config(bin, sh_lmax, bout)) {
    etp_ctx* h = new (std::nothrow) etp_ctx;
    if (!h) {
      set_error("etp_create: out of host memory");
      return ETP_ERR_INVALID_ARG;
    }
    std::string why;
    if (!general_config(bin, sh_lmax, bout, r_cut, &h->c, &why)) {
      delete h;
      set_error("etp_create: unsupported irreps (" + why + ")");
      return ETP_ERR_UNSUPPORTED;
    }
    if (!attach_status_word(h)) {
      delete h;
      return ETP_ERR_CUDA;
    }
    *out = h;
    return ETP_OK;
  }
  const int L = static_cast<int>(bin.size()) - 1;
  const int C = bin[0].mul;
  Ctx c;
  c.lmax = L;
  c.channels = C;
  c.dim = C * (L + 1) * (L + 1);
  c.r_cut = r_cut;
  const std::vector<int> ls = enumerate_paths(bin, sh_lmax, bout);
  bool ok = L == 1 ? fill_from_table<1>(&c, ls) : (L == 2 ? fill_from_table<2>(&c, ls) : fill_from_table<3>(&c, ls));
  if (!ok) {
    set_error("etp_create: path enumeration does not match the generated path tables");
    return ETP_ERR_UNSUPPORTED;
  }
  for (int p = 0; p < c.n_paths; ++p)   // blocks are l = 0..L in order: block index = rank
    for (int k = 0; k < 3; ++k) c.path_blocks[p][k] = static_cast<short>(ls[3 * p + k]);
  etp_ctx* h = new (std::nothrow) etp_ctx;
  if (!h) {
    set_error("etp_create: out of host memory");
    return ETP_ERR_INVALID_ARG;
  }
  c.flop_fwd = 2 * (c.cg_nnz + c.sum_2l3p1) * C;
  c.flop_bwd = 2 * (3 * c.cg_nnz + 2 * c.sum_2l3p1) * C;
  h->c = c;
  if (!attach_status_word(h)) {
    delete h;
    return ETP_ERR_CUDA;
  }
  *out = h;
  return ETP_OK;
}

etp_status etp_get_paths(etp_handle h, int* paths, int capacity) {
  if (!h || (!paths && capacity > 0) || capacity < 0) {
    set_error("etp_get_paths: NULL handle or bad buffer");
    return ETP_ERR_INVALID_ARG;
  }
  if (capacity < h->c.n_paths) {
    set_error("etp_get_paths: capacity " + std::to_string(capacity) + " below the " +
              std::to_string(h->c.n_paths) + " paths");
    return ETP_ERR_CAPACITY;
  }
  for (int p = 0; p < h->c.n_paths; ++p)
    for (int k = 0; k < 3; ++k) paths[3 * p + k] = h->c.path_blocks[p][k];
  return ETP_OK;
}

etp_status etp_destroy(etp_handle h) {
  release_status_word(h);
  delete h;
  return ETP_OK;
}

int* etp_status_word(etp_handle h) { return h ? h->c.status : nullptr; }

etp_status etp_get_status(etp_handle h, void* stream, int* code) {
  if (!h) {
    set_error("etp_get_status: NULL handle");
    return ETP_ERR_INVALID_ARG;
  }
  if (h->c.status_mapped) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_status(e, "etp_get_status: stream synchronisation");
  }
  volatile int* w = reinterpret_cast<volatile int*>(h->c.status);
  const int v = w ? *w : 0;
  if (w) *w = 0;
  if (code) *code = v;
  if (v != 0) {
    set_error("etp_get_status: a bounded pipeline wait gave up (code " + std::to_string(v) +
              "); outputs of the calls since the previous check may be incomplete");
    return ETP_ERR_CUDA;
  }
  return ETP_OK;
}

etp_status etp_get_info(etp_handle h, etp_info_t* info) {
  if (!h || !info) {
    set_error("etp_get_info: NULL argument");
    return ETP_ERR_INVALID_ARG;
  }
  const Ctx& c = h->c;
  info->lmax = c.lmax;
  info->channels = c.channels;
  info->dim_in = c.dim;
  info->dim_out = c.general ? c.gen.dim_out : c.dim;
  info->n_paths = c.n_paths;
  info->n_basis = kNumBasis;
  info->weight_numel = kNumBasis * (c.general ? c.gen.cols : c.n_paths * c.channels);
  info->cg_nnz = c.cg_nnz;
  info->sum_2l3p1 = c.sum_2l3p1;
  info->r_cut = c.r_cut;
  info->general = c.general ? 1 : 0;
  info->flop_fwd = c.flop_fwd;
  info->flop_bwd = c.flop_bwd;
  return ETP_OK;
}

// Workspace: [recv_map: n_edges ints][validation scratch: n_edges + 1 ints][tensor-core forward
// or backward: pre-split weights + status word (+ per-unit edge-gradient partials), or the weight
// gradient's per-edge-range partial sums]
static size_t ws_scratch_offset(int n_edges) { return align256(sizeof(int) * static_cast<size_t>(n_edges)); }
static size_t ws_tc_offset(int n_edges) {
  return ws_scratch_offset(n_edges) + align256(sizeof(int) * (static_cast<size_t>(n_edges) + 1));
}

size_t etp_workspace_bytes(etp_handle h, int n_nodes, int n_edges) {
  if (!h || n_edges < 0 || n_nodes < 0) return 0;
  if (h->c.general) {   // receiver of each edge + validation scratch + edge-gradient or dW partials
    const size_t b = general_backward_partials_bytes(h->c.gen, n_edges);
    const size_t w = general_weight_grad_bytes(h->c.gen, n_edges);
    return ws_tc_offset(n_edges) + (b > w ? b : w);
  }
  const size_t f = tc::forward_tc_workspace_bytes(h->c, n_nodes);
  const size_t b = tc::backward_tc_workspace_bytes(h->c, n_edges);
  const size_t w = weight_grad_workspace_bytes(h->c, n_edges);
  const size_t cxw = cx::workspace_bytes(h->c);
  size_t m = f > b ? f : b;
  m = m > w ? m : w;
  return ws_tc_offset(n_edges) + (m > cxw ? m : cxw);
}

// Forward kernels. By default the channel-major path-subset kernel (etp_fwd_cx.cu) where it
// applies (l_max <= 2, 4 <= C <= 64, C % 4 == 0), else the edge-major tensor-core kernel.
// ETP_FORWARD=edge selects the edge-major kernel and ETP_FORWARD=generic the all-FP32 one. Every
// kernel is tested.
static bool forward_env_is(const char* name) {
  const char* v = std::getenv("ETP_FORWARD");
  return v && std::strcmp(v, name) == 0;
}

static bool use_tc_forward() { return !forward_env_is("generic"); }

static bool use_cx_forward(const Ctx& c) {
  const char* v = std::getenv("ETP_FORWARD");
  return cx::supported(c) && (!v || v[0] == 0 || std::strcmp(v, "default") == 0);
}

// Likewise for the backward: ETP_BACKWARD=generic selects the all-FP32 kernel.
static bool use_tc_backward() {
  const char* v = std::getenv("ETP_BACKWARD");
  return !(v && std::strcmp(v, "generic") == 0);
}

static etp_status check_common(etp_handle h, int n_nodes, int n_edges, const int* row_ptr,
                               const int* sender, const float* edge_vec, const float* x,
                               const float* W, const char* who) {
  if (!h) {
    set_error(std::string(who) + ": NULL handle");
    return ETP_ERR_INVALID_ARG;
  }
  if (n_nodes < 0 || n_edges < 0) {
    set_error(std::string(who) + ": negative size");
    return ETP_ERR_INVALID_ARG;
  }
  const int dmax = h->c.general && h->c.gen.dim_out > h->c.dim ? h->c.gen.dim_out : h->c.dim;
  if (static_cast<long long>(n_nodes) * dmax >= (1LL << 31)) {
    set_error(std::string(who) + ": n_nodes * dim must stay below 2^31");
    return ETP_ERR_UNSUPPORTED;
  }
  if (!row_ptr || (n_edges > 0 && (!sender || !edge_vec || !x || !W))) {
    set_error(std::string(who) + ": NULL array");
    return ETP_ERR_INVALID_ARG;
  }
  if ((x && !aligned16(x)) || (W && !aligned16(W))) {
    set_error(std::string(who) + ": x and W must be 16-byte aligned");
    return ETP_ERR_INVALID_ARG;
  }
  return status_gate(h->c, who);
}

static bool validate_requested() {
  const char* v = std::getenv("ETP_VALIDATE");
  return v && v[0] == '1';
}

etp_status etp_forward(etp_handle h, int n_nodes, int n_edges, const int* row_ptr,
                       const int* sender, const float* edge_vec, const float* x, const float* W,
                       float* out, void* workspace, size_t workspace_bytes, void* stream) {
  etp_status st = check_common(h, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, "etp_forward");
  if (st != ETP_OK) return st;
  if (!out || !aligned16(out)) {
    set_error("etp_forward: out must be a 16-byte aligned device pointer");
    return ETP_ERR_INVALID_ARG;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (validate_requested()) {
    if (!workspace || workspace_bytes < etp_workspace_bytes(h, n_nodes, n_edges)) {
      set_error("etp_forward: ETP_VALIDATE=1 needs the workspace");
      return ETP_ERR_INVALID_ARG;
    }
    int* scratch = reinterpret_cast<int*>(static_cast<char*>(workspace) + ws_scratch_offset(n_edges));
    st = validate_graph(n_nodes, n_edges, row_ptr, sender, nullptr, nullptr, scratch, s);
    if (st != ETP_OK) return st;
  }
  if (n_nodes == 0) return ETP_OK;
  if (h->c.general) {
    st = launch_general_forward(h->c.gen, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, s,
                                h->c.status_dev);
    if (st == ETP_OK && validate_requested()) st = read_status(h->c, s, "general forward");
    return st;
  }
  if (use_tc_forward()) {
    if (!workspace || workspace_bytes < etp_workspace_bytes(h, n_nodes, n_edges)) {
      set_error("etp_forward: workspace missing or smaller than etp_workspace_bytes()");
      return ETP_ERR_INVALID_ARG;
    }
    void* tcws = static_cast<char*>(workspace) + ws_tc_offset(n_edges);
    if (use_cx_forward(h->c)) {
      st = cx::launch(h->c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, tcws, s);
      if (st == ETP_OK && validate_requested()) st = cx::status(h->c, tcws, s);
      return st;
    }
    st = tc::launch_forward_tc(h->c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, tcws, s);
    if (st == ETP_OK && validate_requested()) st = tc::forward_tc_status(h->c, tcws, s);
    return st;
  }
  return launch_forward(h->c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, s);
}

etp_status etp_backward(etp_handle h, int n_nodes, int n_edges, const int* row_ptr,
                        const int* sender, const float* edge_vec, const int* t_row_ptr,
                        const int* t_perm, const float* x, const float* W, const float* grad_out,
                        float* grad_x, float* grad_edge_vec, void* workspace,
                        size_t workspace_bytes, void* stream) {
  etp_status st = check_common(h, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, "etp_backward");
  if (st != ETP_OK) return st;
  if (!t_row_ptr || (n_edges > 0 && (!t_perm || !grad_out)) || (!grad_x && !grad_edge_vec)) {
    set_error("etp_backward: NULL array (grad_x and grad_edge_vec may not both be NULL)");
    return ETP_ERR_INVALID_ARG;
  }
  if ((grad_x && !aligned16(grad_x)) || (grad_out && !aligned16(grad_out))) {
    set_error("etp_backward: grad_x and grad_out must be 16-byte aligned");
    return ETP_ERR_INVALID_ARG;
  }
  if (n_edges > 0 && (!workspace || workspace_bytes < etp_workspace_bytes(h, n_nodes, n_edges))) {
    set_error("etp_backward: workspace missing or smaller than etp_workspace_bytes()");
    return ETP_ERR_INVALID_ARG;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* recv_map = static_cast<int*>(workspace);
  if (validate_requested()) {
    int* scratch = reinterpret_cast<int*>(static_cast<char*>(workspace) + ws_scratch_offset(n_edges));
    st = validate_graph(n_nodes, n_edges, row_ptr, sender, t_row_ptr, t_perm, scratch, s);
    if (st != ETP_OK) return st;
  }
  if (n_nodes == 0) return ETP_OK;
  if (h->c.general)
    return launch_general_backward(h->c.gen, n_nodes, n_edges, row_ptr, edge_vec, t_row_ptr, t_perm, x, W,
                                   grad_out, grad_x, grad_edge_vec, recv_map,
                                   reinterpret_cast<float*>(static_cast<char*>(workspace) + ws_tc_offset(n_edges)),
                                   s);
  if (n_edges > 0 && use_tc_backward()) {
    void* tcws = static_cast<char*>(workspace) + ws_tc_offset(n_edges);
    st = tc::launch_backward_tc(h->c, n_nodes, n_edges, row_ptr, edge_vec, t_row_ptr, t_perm, x, W, grad_out,
                                grad_x, grad_edge_vec, recv_map, tcws, s);
    if (st == ETP_OK && validate_requested()) st = tc::backward_tc_status(h->c, tcws, s);
    return st;
  }
  return launch_backward(h->c, n_nodes, n_edges, row_ptr, sender, edge_vec, t_row_ptr, t_perm, x,
                         W, grad_out, grad_x, grad_edge_vec, recv_map, s);
}

etp_status etp_forward_masked(etp_handle h, int n_nodes, int n_edges, const int* row_ptr,
                              const int* sender, const float* edge_vec, const float* x, const float* W,
                              const uint32_t* path_mask, float* out, void* workspace,
                              size_t workspace_bytes, void* stream) {
  etp_status st = check_common(h, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, "etp_forward_masked");
  if (st != ETP_OK) return st;
  if (h->c.general && h->c.n_paths > 32) {
    set_error("etp_forward_masked: a 32-bit path mask covers at most 32 paths");
    return ETP_ERR_UNSUPPORTED;
  }
  if (!out || !aligned16(out) || (n_edges > 0 && !path_mask)) {
    set_error("etp_forward_masked: out (16-byte aligned) and path_mask must be device pointers");
    return ETP_ERR_INVALID_ARG;
  }
  if (!workspace || workspace_bytes < etp_workspace_bytes(h, n_nodes, n_edges)) {
    set_error("etp_forward_masked: workspace missing or smaller than etp_workspace_bytes()");
    return ETP_ERR_INVALID_ARG;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (validate_requested()) {
    int* scratch = reinterpret_cast<int*>(static_cast<char*>(workspace) + ws_scratch_offset(n_edges));
    st = validate_graph(n_nodes, n_edges, row_ptr, sender, nullptr, nullptr, scratch, s);
    if (st != ETP_OK) return st;
  }
  if (n_nodes == 0) return ETP_OK;
  if (h->c.general)
    return launch_general_forward(h->c.gen, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, s,
                                  h->c.status_dev, n_edges > 0 ? path_mask : nullptr);
  void* tcws = static_cast<char*>(workspace) + ws_tc_offset(n_edges);
  st = tc::launch_forward_tc(h->c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, out, tcws, s,
                             n_edges > 0 ? path_mask : nullptr);
  if (st == ETP_OK && validate_requested()) st = tc::forward_tc_status(h->c, tcws, s);
  return st;
}

etp_status etp_backward_masked(etp_handle h, int n_nodes, int n_edges, const int* row_ptr,
                               const int* sender, const float* edge_vec, const int* t_row_ptr,
                               const int* t_perm, const float* x, const float* W,
                               const uint32_t* path_mask, const float* grad_out, float* grad_x,
                               float* grad_edge_vec, void* workspace, size_t workspace_bytes,
                               void* stream) {
  etp_status st = check_common(h, n_nodes, n_edges, row_ptr, sender, edge_vec, x, W, "etp_backward_masked");
  if (st != ETP_OK) return st;
  if (h->c.general && h->c.n_paths > 32) {
    set_error("etp_backward_masked: a 32-bit path mask covers at most 32 paths");
    return ETP_ERR_UNSUPPORTED;
  }
  if (!t_row_ptr || (n_edges > 0 && (!t_perm || !grad_out || !path_mask)) || (!grad_x && !grad_edge_vec)) {
    set_error("etp_backward_masked: NULL array (grad_x and grad_edge_vec may not both be NULL)");
    return ETP_ERR_INVALID_ARG;
  }
  if ((grad_x && !aligned16(grad_x)) || (grad_out && !aligned16(grad_out))) {
    set_error("etp_backward_masked: grad_x and grad_out must be 16-byte aligned");
    return ETP_ERR_INVALID_ARG;
  }
  if (!workspace || workspace_bytes < etp_workspace_bytes(h, n_nodes, n_edges)) {
    set_error("etp_backward_masked: workspace missing or smaller than etp_workspace_bytes()");
    return ETP_ERR_INVALID_ARG;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (validate_requested()) {
    int* scratch = reinterpret_cast<int*>(static_cast<char*>(workspace) + ws_scratch_offset(n_edges));
    st = validate_graph(n_nodes, n_edges, row_ptr, sender, t_row_ptr, t_perm, scratch, s);
    if (st != ETP_OK) return st;
  }
  if (n_nodes == 0) return ETP_OK;
  if (h->c.general)
    return launch_general_backward(h->c.gen, n_nodes, n_edges, row_ptr, edge_vec, t_row_ptr, t_perm, x, W,
                                   grad_out, grad_x, grad_edge_vec, static_cast<int*>(workspace),
                                   reinterpret_cast<float*>(static_cast<char*>(workspace) + ws_tc_offset(n_edges)),
                                   s, n_edges > 0 ? path_mask : nullptr);
  if (n_edges == 0)   // nothing is sent: zero outputs from the kernel without edges
    return launch_backward(h->c, n_nodes, n_edges, row_ptr, sender, edge_vec, t_row_ptr, t_perm, x, W, grad_out,
                           grad_x, grad_edge_vec, static_cast<int*>(workspace), s);
  void* tcws = static_cast<char*>(workspace) + ws_tc_offset(n_edges);
  st = tc::launch_backward_tc(h->c, n_nodes, n_edges, row_ptr, edge_vec, t_row_ptr, t_perm, x, W, grad_out, grad_x,
                              grad_edge_vec, static_cast<int*>(workspace), tcws, s, path_mask);
  if (st == ETP_OK && validate_requested()) st = tc::backward_tc_status(h->c, tcws, s);
  return st;
}

etp_status etp_backward_weights(etp_handle h, int n_nodes, int n_edges, const int* row_ptr,
                                const int* sender, const float* edge_vec, const float* x,
                                const float* grad_out, float* grad_W, void* workspace,
                                size_t workspace_bytes, void* stream) {
  if (!h) {
    set_error("etp_backward_weights: NULL handle");
    return ETP_ERR_INVALID_ARG;
  }

  if (n_nodes < 0 || n_edges < 0) {
    set_error("etp_backward_weights: negative size");
    return ETP_ERR_INVALID_ARG;
  }
  if (static_cast<long long>(n_nodes) * h->c.dim >= (1LL << 31)) {
    set_error("etp_backward_weights: n_nodes * dim must stay below 2^31");
    return ETP_ERR_UNSUPPORTED;
  }
  if (!row_ptr || !grad_W || (n_edges > 0 && (!sender || !edge_vec || !x || !grad_out))) {
    set_error("etp_backward_weights: NULL array");
    return ETP_ERR_INVALID_ARG;
  }
  if (n_edges > 0 && (!workspace || workspace_bytes < etp_workspace_bytes(h, n_nodes, n_edges))) {
    set_error("etp_backward_weights: workspace missing or smaller than etp_workspace_bytes()");
    return ETP_ERR_INVALID_ARG;
  }
  if (status_gate(h->c, "etp_backward_weights") != ETP_OK) return ETP_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (validate_requested() && n_edges > 0) {
    int* scratch = reinterpret_cast<int*>(static_cast<char*>(workspace) + ws_scratch_offset(n_edges));
    etp_status st = validate_graph(n_nodes, n_edges, row_ptr, sender, nullptr, nullptr, scratch, s);
    if (st != ETP_OK) return st;
  }
  int* recv = static_cast<int*>(workspace);
  void* part = workspace ? static_cast<char*>(workspace) + ws_tc_offset(n_edges) : nullptr;
  if (h->c.general)
    return launch_general_weight_grad(h->c.gen, n_nodes, n_edges, row_ptr, sender, edge_vec, x, grad_out, grad_W,
                                      recv, static_cast<float*>(part), s);
  return launch_weight_grad(h->c, n_nodes, n_edges, row_ptr, sender, edge_vec, x, grad_out, grad_W, recv, part, s);
}

etp_status etp_node_ladder(int lmax, int channels, int n_nodes, int nu, const float* A, const float* W,
                           float* out, void* stream) {
  if (lmax < 1 || lmax > kMaxL) {
    set_error("etp_node_ladder: lmax must be 1, 2 or 3");
    return ETP_ERR_UNSUPPORTED;
  }
  if (channels < 4 || channels > 256 || channels % 4 != 0) {
    set_error("etp_node_ladder: channels must be a multiple of 4 in [4, 256]");
    return ETP_ERR_UNSUPPORTED;
  }
  if (n_nodes < 0 || nu < 1 || nu > 8) {
    set_error("etp_node_ladder: n_nodes >= 0 and 1 <= nu <= 8");
    return ETP_ERR_INVALID_ARG;
  }
  if (static_cast<long long>(n_nodes) * (lmax + 1) * (lmax + 1) * channels >= (1LL << 31)) {
    set_error("etp_node_ladder: n_nodes * dim must stay below 2^31");
    return ETP_ERR_UNSUPPORTED;
  }
  if (n_nodes > 0 && (!A || !out || (nu > 1 && !W))) {
    set_error("etp_node_ladder: NULL array");
    return ETP_ERR_INVALID_ARG;
  }
  if ((A && !aligned16(A)) || (out && !aligned16(out)) || (W && !aligned16(W))) {
    set_error("etp_node_ladder: A, W and out must be 16-byte aligned");
    return ETP_ERR_INVALID_ARG;
  }
  if (n_nodes == 0) return ETP_OK;
  return launch_node_ladder(lmax, channels, n_nodes, nu, A, W, out, static_cast<cudaStream_t>(stream));
}

size_t etp_node_ladder_full_step_floats(int lmax, int channels) {
  return lad::supported(lmax, channels) ? lad::step_weight_floats(lmax, channels) : 0;
}

size_t etp_node_ladder_full_workspace_bytes(int lmax, int channels, int n_nodes) {
  return lad::workspace_bytes(lmax, channels, n_nodes);
}

etp_status etp_node_ladder_full(int lmax, int channels, int n_nodes, int nu, const float* A, const float* W,
                                float* out, void* workspace, size_t workspace_bytes, void* stream) {
  if (!lad::supported(lmax, channels)) {
    set_error("etp_node_ladder_full: lmax must be 1, 2 or 3 and channels 32, 64, 96 or 128");
    return ETP_ERR_UNSUPPORTED;
  }
  if (n_nodes < 0 || nu < 1 || nu > 8) {
    set_error("etp_node_ladder_full: n_nodes >= 0 and 1 <= nu <= 8");
    return ETP_ERR_INVALID_ARG;
  }
  if (static_cast<long long>(n_nodes) * 99 * channels >= (1LL << 40)) {
    set_error("etp_node_ladder_full: too many nodes");
    return ETP_ERR_UNSUPPORTED;
  }
  if (n_nodes > 0 && (!A || !out || (nu > 1 && !W))) {
    set_error("etp_node_ladder_full: NULL array");
    return ETP_ERR_INVALID_ARG;
  }
  if ((A && !aligned16(A)) || (out && !aligned16(out)) || (W && !aligned16(W))) {
    set_error("etp_node_ladder_full: A, W and out must be 16-byte aligned");
    return ETP_ERR_INVALID_ARG;
  }
  if (n_nodes == 0) return ETP_OK;
  if (!workspace || workspace_bytes < lad::workspace_bytes(lmax, channels, n_nodes) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) {
    set_error("etp_node_ladder_full: workspace missing, misaligned or smaller than "
              "etp_node_ladder_full_workspace_bytes()");
    return ETP_ERR_INVALID_ARG;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = nullptr;
  etp_status st = lad::launch(lmax, channels, nu, n_nodes, A, W, out, workspace, s, &status);
  if (st != ETP_OK || !validate_requested()) return st;
  int code = 0;
  cudaError_t e = cudaMemcpyAsync(&code, status, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_status(e, "etp_node_ladder_full status");
  if (code != 0) {
    set_error("etp_node_ladder_full: a tensor-core pipeline wait gave up (code " + std::to_string(code) + ")");
    return ETP_ERR_CUDA;
  }
  return ETP_OK;
}

etp_status etp_radial_weights(etp_handle h, int n_edges, const float* edge_vec, const float* W,
                              float* w_out, void* stream) {
  if (!h || n_edges < 0 || (n_edges > 0 && (!edge_vec || !W || !w_out))) {
    set_error("etp_radial_weights: bad argument");
    return ETP_ERR_INVALID_ARG;
  }
  if (h->c.general) {
    set_error("etp_radial_weights: not implemented for general irreps handles");
    return ETP_ERR_UNSUPPORTED;
  }
  if (status_gate(h->c, "etp_radial_weights") != ETP_OK) return ETP_ERR_CUDA;
  if (n_edges == 0) return ETP_OK;
  return launch_radial_weights(h->c, n_edges, edge_vec, W, w_out, static_cast<cudaStream_t>(stream));
}

etp_status etp_forces(int n_nodes, int n_edges, const int* row_ptr, const int* t_row_ptr,
                      const int* t_perm, const float* grad_edge_vec, float* forces, void* stream) {
  if (n_nodes < 0 || n_edges < 0 || !row_ptr || !t_row_ptr || !forces ||
      (n_edges > 0 && (!t_perm || !grad_edge_vec))) {
    set_error("etp_forces: bad argument");
    return ETP_ERR_INVALID_ARG;
  }
  if (n_nodes == 0) return ETP_OK;
  return launch_forces(n_nodes, n_edges, row_ptr, t_row_ptr, t_perm, grad_edge_vec, forces,
                       static_cast<cudaStream_t>(stream));
}

size_t etp_graph_workspace_bytes(int n_nodes, int max_edges) {
  if (n_nodes < 0 || max_edges < 0) return 0;
  return graph_workspace_bytes(n_nodes, max_edges);
}

etp_status etp_neighbors(const float* pos, int n_nodes, const double* cell, const int* pbc,
                         float r_cut, int max_edges, int* n_edges, int* row_ptr, int* sender,
                         float* edge_vec, int* shift, int* t_row_ptr, int* t_perm,
                         void* workspace, size_t workspace_bytes, void* stream) {
  if (n_nodes < 0 || max_edges < 0 || !n_edges || !row_ptr || !t_row_ptr || !(r_cut > 0.f) ||
      (n_nodes > 0 && !pos) || (max_edges > 0 && (!sender || !edge_vec || !t_perm))) {
    set_error("etp_neighbors: bad argument");
    return ETP_ERR_INVALID_ARG;
  }
  if (workspace_bytes < graph_workspace_bytes(n_nodes, max_edges) || (!workspace && workspace_bytes)) {
    set_error("etp_neighbors: workspace smaller than etp_graph_workspace_bytes()");
    return ETP_ERR_INVALID_ARG;
  }
  return neighbors(pos, n_nodes, cell, pbc, r_cut, max_edges, n_edges, row_ptr, sender, edge_vec,
                   shift, t_row_ptr, t_perm, workspace, workspace_bytes,
                   static_cast<cudaStream_t>(stream));
}

etp_status etp_build_csr(int n_nodes, int n_edges, const int* receiver, const int* sender_in,
                         const float* edge_vec_in, int* row_ptr, int* sender, float* edge_vec,
                         int* perm, int* t_row_ptr, int* t_perm, void* workspace,
                         size_t workspace_bytes, void* stream) {
  if (n_nodes < 0 || n_edges < 0 || !row_ptr || !t_row_ptr ||
      (n_edges > 0 && (!receiver || !sender_in || !edge_vec_in || !sender || !edge_vec || !t_perm))) {
    set_error("etp_build_csr: bad argument");
    return ETP_ERR_INVALID_ARG;
  }
  if (workspace_bytes < graph_workspace_bytes(n_nodes, n_edges) || (!workspace && workspace_bytes)) {
    set_error("etp_build_csr: workspace smaller than etp_graph_workspace_bytes()");
    return ETP_ERR_INVALID_ARG;
  }
  return build_csr(n_nodes, n_edges, receiver, sender_in, edge_vec_in, row_ptr, sender, edge_vec,
                   perm, t_row_ptr, t_perm, workspace, workspace_bytes,
                   static_cast<cudaStream_t>(stream));
}

}  // extern "C"
