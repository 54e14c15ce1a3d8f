// C ABI of libcgtp.so: argument checks, plans, coefficient-table upload and
// dispatch to the per-shape kernels.  Declared in include/cgtp.h.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <new>
#include <vector>

#include "cg_table.h"
#include "configs.h"
#include "launch.h"
#include "structure.h"
#include "../../include/cgtp.h"

namespace cgtp {

// ---------------------------------------------------------------- uploaders
static std::vector<UploadFn>& uploaders() {
  static std::vector<UploadFn> v;
  return v;
}
int register_table_uploader(UploadFn fn) {
  uploaders().push_back(fn);
  return 1;
}

namespace {

thread_local int g_last_cuda_error = 0;

cgtp_status cuda_fail(cudaError_t e) {
  g_last_cuda_error = (int)e;
  return CGTP_ERR_CUDA;
}

struct HostTables {
  float cg[kTableSize];
  float shk[kShkSize];
  int status = -1;
};

HostTables& host_tables() {
  static HostTables t;
  static std::once_flag once;
  std::call_once(once, [] { t.status = build_constant_tables(t.cg, t.shk); });
  return t;
}

std::mutex g_dev_mutex;
std::vector<int> g_uploaded;  // per device: 1 once the tables are in its constant memory
std::vector<int> g_num_sms;

cgtp_status ensure_device(int* num_sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  if ((int)g_uploaded.size() <= dev) {
    g_uploaded.resize(dev + 1, 0);
    g_num_sms.resize(dev + 1, 0);
  }
  if (!g_uploaded[dev]) {
    HostTables& t = host_tables();
    if (t.status != 0) return CGTP_ERR_TABLE;
    for (UploadFn fn : uploaders()) {
      e = fn(t.cg, t.shk);
      if (e != cudaSuccess) return cuda_fail(e);
    }
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    g_num_sms[dev] = sms;
    g_uploaded[dev] = 1;
  }
  *num_sms = g_num_sms[dev];
  return CGTP_OK;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

#define CGTP_LIST_ENTRY(a, b, c) {a, b, c},
struct Shape {
  int li, ls, lo;
};
const Shape kShapes[] = {CGTP_CONFIGS(CGTP_LIST_ENTRY)};
const Shape kVariantShapes[] = {CGTP_VARIANT_CONFIGS(CGTP_LIST_ENTRY)};

template <size_t N>
bool listed(const Shape (&list)[N], int li, int ls, int lo) {
  for (const Shape& s : list)
    if (s.li == li && s.ls == ls && s.lo == lo) return true;
  return false;
}

}  // namespace
}  // namespace cgtp

using namespace cgtp;

struct cgtp_plan_s {
  int li, ls, lo, mult;
  cgtp_mode mode;
  int n_paths;
  int nnz;
  std::vector<int> paths;
  // checked mode: validation flags on the device of cgtp_plan_set_checked
  int checked = 0;
  int* d_flags = nullptr;
  int flags_device = -1;
};

namespace {

bool mode_is(cgtp_plan p, cgtp_mode m) { return p != nullptr && p->mode == m; }
bool conv_mode(cgtp_plan p) {  // plans whose convolution takes one weight row per path or one shared row
  return p != nullptr && (p->mode == CGTP_MODE_CONV_UVU || p->mode == CGTP_MODE_CONV_UVU_SHARED);
}

// Checked mode: OR the validation bits of the graph arrays a call uses into
// the plan's flags (same stream, before the call's kernels) and hand the
// flags to the kernels, which do nothing when they mark the graph unsafe.
cudaError_t validate_graph(cgtp_plan p, int n, int E, const int* row_ptr, const int* col, const float* edge_vec,
                           const int* csc_ptr, const int* csc_edge, const int* csc_dst, int sms, cudaStream_t s,
                           const int** abort_flag) {
  *abort_flag = nullptr;
  if (!p->checked) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev != p->flags_device) return cudaErrorInvalidDevice;
  *abort_flag = p->d_flags;
  return launch_graph_validate(n, E, row_ptr, col, edge_vec, csc_ptr, csc_edge, csc_dst, p->d_flags, sms, s);
}

}  // namespace

extern "C" {

const char* cgtp_status_string(cgtp_status s) {
  switch (s) {
    case CGTP_OK: return "CGTP_OK";
    case CGTP_ERR_INVALID_ARG: return "CGTP_ERR_INVALID_ARG";
    case CGTP_ERR_UNSUPPORTED: return "CGTP_ERR_UNSUPPORTED";
    case CGTP_ERR_BAD_GRAPH: return "CGTP_ERR_BAD_GRAPH";
    case CGTP_ERR_OOM: return "CGTP_ERR_OOM";
    case CGTP_ERR_CUDA: return "CGTP_ERR_CUDA";
    case CGTP_ERR_TABLE: return "CGTP_ERR_TABLE";
    case CGTP_ERR_WORKSPACE: return "CGTP_ERR_WORKSPACE";
  }
  return "CGTP_ERR_UNKNOWN";
}

int cgtp_last_cuda_error(void) { return g_last_cuda_error; }

int cgtp_supported(int li, int ls, int lo, cgtp_mode mode) {
  switch (mode) {
    case CGTP_MODE_CONV_UVU:
    case CGTP_MODE_PAIR_UVU: return listed(kShapes, li, ls, lo) ? 1 : 0;
    case CGTP_MODE_CONV_UVU_SHARED:
    case CGTP_MODE_CONV_UVW: return listed(kVariantShapes, li, ls, lo) ? 1 : 0;
  }
  return 0;
}

cgtp_status cgtp_cg_block(int l1, int l2, int l3, double* out) {
  if (out == nullptr || l1 < 0 || l2 < 0 || l3 < 0 || l1 > kLmaxTab || l2 > kLmaxTab || l3 > kLmaxTab)
    return CGTP_ERR_INVALID_ARG;
  double disc = 0.0;
  real_cg_block(l1, l2, l3, out, &disc);
  return disc > 1e-12 ? CGTP_ERR_TABLE : CGTP_OK;
}

cgtp_status cgtp_plan_create(int li, int ls, int lo, int mult, cgtp_mode mode, cgtp_plan* plan) {
  if (plan == nullptr) return CGTP_ERR_INVALID_ARG;
  *plan = nullptr;
  if (li < 0 || ls < 0 || lo < 0 || mult <= 0 || mult % 4 != 0) return CGTP_ERR_INVALID_ARG;
  if (mode != CGTP_MODE_CONV_UVU && mode != CGTP_MODE_PAIR_UVU && mode != CGTP_MODE_CONV_UVU_SHARED &&
      mode != CGTP_MODE_CONV_UVW)
    return CGTP_ERR_INVALID_ARG;
  if (!cgtp_supported(li, ls, lo, mode)) return CGTP_ERR_UNSUPPORTED;
  if (host_tables().status != 0) return CGTP_ERR_TABLE;
  int sms = 0;
  cgtp_status st = ensure_device(&sms);
  if (st != CGTP_OK) return st;
  cgtp_plan_s* p = new (std::nothrow) cgtp_plan_s();
  if (p == nullptr) return CGTP_ERR_OOM;
  const PathData d = make_paths(li, ls, lo);
  p->li = li;
  p->ls = ls;
  p->lo = lo;
  p->mult = mult;
  p->mode = mode;
  p->n_paths = d.np;
  p->nnz = d.nnz;
  for (int k = 0; k < d.np; ++k) {
    p->paths.push_back(d.l1[k]);
    p->paths.push_back(d.l2[k]);
    p->paths.push_back(d.l3[k]);
  }
  *plan = p;
  return CGTP_OK;
}

cgtp_status cgtp_plan_destroy(cgtp_plan plan) {
  if (plan != nullptr && plan->d_flags != nullptr) {
    int cur = 0;
    if (cudaGetDevice(&cur) == cudaSuccess && cudaSetDevice(plan->flags_device) == cudaSuccess) {
      cudaFree(plan->d_flags);
      cudaSetDevice(cur);
    }
  }
  delete plan;
  return CGTP_OK;
}

cgtp_status cgtp_plan_set_checked(cgtp_plan plan, int checked) {
  if (plan == nullptr) return CGTP_ERR_INVALID_ARG;
  if (checked && plan->d_flags == nullptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaMalloc(&plan->d_flags, 16);
    if (e == cudaSuccess) e = cudaMemset(plan->d_flags, 0, 16);
    if (e != cudaSuccess) {
      if (plan->d_flags) cudaFree(plan->d_flags);
      plan->d_flags = nullptr;
      return e == cudaErrorMemoryAllocation ? CGTP_ERR_OOM : cuda_fail(e);
    }
    plan->flags_device = dev;
  }
  plan->checked = checked ? 1 : 0;
  return CGTP_OK;
}

cgtp_status cgtp_plan_check(cgtp_plan plan, int* flags) {
  if (plan == nullptr) return CGTP_ERR_INVALID_ARG;
  if (flags) *flags = 0;
  if (plan->d_flags == nullptr) return CGTP_OK;  // never in checked mode: nothing recorded
  int cur = 0;
  cudaError_t e = cudaGetDevice(&cur);
  if (e == cudaSuccess) e = cudaSetDevice(plan->flags_device);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  int f = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&f, plan->d_flags, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(plan->d_flags, 0, sizeof(int));
  cudaSetDevice(cur);
  if (e != cudaSuccess) return cuda_fail(e);
  if (flags) *flags = f;
  return f ? CGTP_ERR_BAD_GRAPH : CGTP_OK;
}

cgtp_status cgtp_plan_info(cgtp_plan plan, int* n_paths, int* paths, int* n_nonzero) {
  if (plan == nullptr) return CGTP_ERR_INVALID_ARG;
  if (n_paths) *n_paths = plan->n_paths;
  if (paths)
    for (size_t k = 0; k < plan->paths.size(); ++k) paths[k] = plan->paths[k];
  if (n_nonzero) *n_nonzero = plan->nnz;
  return CGTP_OK;
}

cgtp_status cgtp_graph_build(const float* pos, int n, float box_len, float rc, const int* graph_ptr,
                             int n_graphs, int* row_ptr, int* col, float* edge_vec, int* csc_ptr,
                             int* csc_edge, int* csc_dst, int max_edges, int* n_edges, void* stream) {
  if (n < 0 || max_edges < 0 || !(rc > 0.f) || row_ptr == nullptr || csc_ptr == nullptr || n_edges == nullptr)
    return CGTP_ERR_INVALID_ARG;
  if (n > 0 && pos == nullptr) return CGTP_ERR_INVALID_ARG;
  if (max_edges > 0 && (col == nullptr || edge_vec == nullptr || csc_edge == nullptr || csc_dst == nullptr))
    return CGTP_ERR_INVALID_ARG;
  if (graph_ptr != nullptr && n_graphs < 1) return CGTP_ERR_INVALID_ARG;
  if (box_len > 0.f && !((double)rc < 0.5 * (double)box_len)) return CGTP_ERR_INVALID_ARG;
  int sms = 0;
  cgtp_status st = ensure_device(&sms);
  if (st != CGTP_OK) return st;
  cudaError_t e = launch_graph_build(pos, n, box_len, rc, graph_ptr, n_graphs, row_ptr, col, edge_vec, csc_ptr,
                                     csc_edge, csc_dst, max_edges, n_edges, sms, (cudaStream_t)stream);
  return e == cudaSuccess ? CGTP_OK : cuda_fail(e);
}

cgtp_status cgtp_csr_transpose(int n, int n_edges, const int* row_ptr, const int* col, int* csc_ptr, int* csc_edge,
                               int* csc_dst, void* workspace, size_t workspace_bytes, void* stream) {
  if (n < 0 || n_edges < 0 || row_ptr == nullptr || csc_ptr == nullptr) return CGTP_ERR_INVALID_ARG;
  if (n_edges > 0 && (col == nullptr || csc_edge == nullptr || csc_dst == nullptr)) return CGTP_ERR_INVALID_ARG;
  if (workspace == nullptr || workspace_bytes < sizeof(int) * (size_t)(n > 0 ? n : 1)) return CGTP_ERR_WORKSPACE;
  int sms = 0;
  cgtp_status st = ensure_device(&sms);
  if (st != CGTP_OK) return st;
  cudaError_t e = launch_csr_transpose(n, n_edges, row_ptr, col, csc_ptr, csc_edge, csc_dst, (int*)workspace, sms,
                                       (cudaStream_t)stream);
  return e == cudaSuccess ? CGTP_OK : cuda_fail(e);
}

cgtp_status cgtp_graph_check(int n, int n_edges, const int* row_ptr, const int* col, const float* edge_vec,
                             int* flags, void* stream) {
  if (n < 0 || n_edges < 0 || row_ptr == nullptr || flags == nullptr) return CGTP_ERR_INVALID_ARG;
  if (n_edges > 0 && (col == nullptr || edge_vec == nullptr)) return CGTP_ERR_INVALID_ARG;
  int sms = 0;
  cgtp_status st = ensure_device(&sms);
  if (st != CGTP_OK) return st;
  cudaError_t e = launch_graph_check(n, n_edges, row_ptr, col, edge_vec, flags, sms, (cudaStream_t)stream);
  return e == cudaSuccess ? CGTP_OK : cuda_fail(e);
}

cgtp_status cgtp_spherical_harmonics(int lmax_sh, int n_edges, const float* edge_vec, float* Y, float* dY,
                                     void* stream) {
  if (lmax_sh < 0 || lmax_sh > kLmaxTab || n_edges < 0) return CGTP_ERR_INVALID_ARG;
  if (n_edges > 0 && (edge_vec == nullptr || (Y == nullptr && dY == nullptr))) return CGTP_ERR_INVALID_ARG;
  int sms = 0;
  cgtp_status st = ensure_device(&sms);
  if (st != CGTP_OK) return st;
  cudaError_t e = launch_sh(lmax_sh, n_edges, edge_vec, Y, dY, sms, (cudaStream_t)stream);
  return e == cudaSuccess ? CGTP_OK : cuda_fail(e);
}

cgtp_status cgtp_conv_forward(cgtp_plan p, int n_nodes, int n_edges, const int* row_ptr, const int* col,
                              const float* edge_vec, const float* x, const float* w, float* out, void* stream) {
  if (!conv_mode(p) || n_nodes < 0 || n_edges < 0 || row_ptr == nullptr) return CGTP_ERR_INVALID_ARG;
  if (n_nodes > 0 && (x == nullptr || out == nullptr)) return CGTP_ERR_INVALID_ARG;
  if (n_edges > 0 && (col == nullptr || edge_vec == nullptr || w == nullptr)) return CGTP_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(out)) return CGTP_ERR_INVALID_ARG;
  if (n_nodes == 0) return CGTP_OK;
  int sms = 0;
  cgtp_status st = ensure_device(&sms);
  if (st != CGTP_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  ConvFwdArgs a{n_nodes, row_ptr, col, edge_vec, x, w, out, p->mult};
  cudaError_t e = validate_graph(p, n_nodes, n_edges, row_ptr, col, edge_vec, nullptr, nullptr, nullptr, sms, s,
                                 &a.abort_flag);
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaErrorNotSupported;
  if (p->mode == CGTP_MODE_CONV_UVU_SHARED) {
#define CGTP_SFWD_ENTRY(A, B, C) \
    if (p->li == A && p->ls == B && p->lo == C) e = launch_conv_fwd_shared<A, B, C>(a, sms, s);
    CGTP_VARIANT_CONFIGS(CGTP_SFWD_ENTRY)
  } else {
#define CGTP_FWD_ENTRY(A, B, C) \
    if (p->li == A && p->ls == B && p->lo == C) e = launch_conv_fwd<A, B, C>(a, sms, s);
    CGTP_CONFIGS(CGTP_FWD_ENTRY)
  }
  return e == cudaSuccess ? CGTP_OK : cuda_fail(e);
}

static int bwd_slices(cgtp_plan p) {
  int s = 0;
#define CGTP_SLICES_ENTRY(A, B, C) \
  if (p->li == A && p->ls == B && p->lo == C) s = conv_bwd_slices<A, B, C>(p->mult);
  CGTP_CONFIGS(CGTP_SLICES_ENTRY)
  return s;
}

cgtp_status cgtp_conv_backward_workspace_size(cgtp_plan p, int n_edges, size_t* bytes) {
  if (p == nullptr || p->mode == CGTP_MODE_PAIR_UVU || n_edges < 0 || bytes == nullptr) return CGTP_ERR_INVALID_ARG;
  const size_t ns = (size_t)(p->ls + 1) * (p->ls + 1);
  const size_t b = sizeof(float) * (size_t)bwd_slices(p) * (size_t)n_edges * ns;
  *bytes = (b + 255) & ~(size_t)255;
  return CGTP_OK;
}

cgtp_status cgtp_conv_backward(cgtp_plan p, int n_nodes, int n_edges, const int* csc_ptr, const int* csc_edge,
                               const int* csc_dst, const float* edge_vec, const float* x, const float* w,
                               const float* grad_out, float* grad_x, float* grad_w, float* grad_edge_vec,
                               void* workspace, size_t workspace_bytes, void* stream) {
  if (!conv_mode(p) || n_nodes < 0 || n_edges < 0 || csc_ptr == nullptr) return CGTP_ERR_INVALID_ARG;
  if (n_nodes > 0 && (x == nullptr || grad_out == nullptr)) return CGTP_ERR_INVALID_ARG;
  if (n_edges > 0 && (csc_edge == nullptr || csc_dst == nullptr || edge_vec == nullptr || w == nullptr))
    return CGTP_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(grad_out) || !aligned16(grad_x) || !aligned16(grad_w))
    return CGTP_ERR_INVALID_ARG;
  if (grad_edge_vec != nullptr && n_edges > 0) {
    size_t need = 0;
    cgtp_conv_backward_workspace_size(p, n_edges, &need);
    if (workspace == nullptr || workspace_bytes < need || ((uintptr_t)workspace & 255u) != 0)
      return CGTP_ERR_WORKSPACE;
  }
  int sms = 0;
  cgtp_status st = ensure_device(&sms);
  if (st != CGTP_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (n_nodes == 0) return CGTP_OK;
  if (n_edges == 0) {  // no edges: every gradient is zero
    cudaError_t e = cudaSuccess;
    if (grad_x) e = cudaMemsetAsync(grad_x, 0, sizeof(float) * (size_t)n_nodes * (p->li + 1) * (p->li + 1) * p->mult, s);
    return e == cudaSuccess ? CGTP_OK : cuda_fail(e);
  }
  ConvBwdArgs a{n_nodes, n_edges, csc_ptr, csc_edge, csc_dst, edge_vec, x, w, grad_out,
                grad_x, grad_w, grad_edge_vec, (float*)workspace, p->mult};
  cudaError_t e = validate_graph(p, n_nodes, n_edges, nullptr, nullptr, edge_vec, csc_ptr, csc_edge, csc_dst, sms, s,
                                 &a.abort_flag);
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaErrorNotSupported;
  if (p->mode == CGTP_MODE_CONV_UVU_SHARED) {
#define CGTP_SBWD_ENTRY(A, B, C) \
    if (p->li == A && p->ls == B && p->lo == C) e = launch_conv_bwd_shared<A, B, C>(a, sms, s);
    CGTP_VARIANT_CONFIGS(CGTP_SBWD_ENTRY)
  } else {
#define CGTP_BWD_ENTRY(A, B, C) \
    if (p->li == A && p->ls == B && p->lo == C) e = launch_conv_bwd<A, B, C>(a, sms, s);
    CGTP_CONFIGS(CGTP_BWD_ENTRY)
  }
  return e == cudaSuccess ? CGTP_OK : cuda_fail(e);
}

// ---- double backward: the adjoint of cgtp_conv_backward ----
static cudaError_t dispatch_fwd(cgtp_plan p, const ConvFwdArgs& a, int sms, cudaStream_t s) {
  cudaError_t e = cudaErrorNotSupported;
#define CGTP_DFWD_ENTRY(A, B, C) \
  if (p->li == A && p->ls == B && p->lo == C) e = launch_conv_fwd<A, B, C>(a, sms, s);
  CGTP_CONFIGS(CGTP_DFWD_ENTRY)
  return e;
}
static cudaError_t dispatch_bwd(cgtp_plan p, const ConvBwdArgs& a, int sms, cudaStream_t s);
// Harmonic-gradient pass of the first-order double backward: the plain
// backward with neither grad_x nor grad_W requested (nothing but the grad_Y
// partials and the Jacobian epilogue of a.gr_mode is written).
static cudaError_t dispatch_bwd_gy(cgtp_plan p, const ConvBwdArgs& a, int sms, cudaStream_t s) {
  return dispatch_bwd(p, a, sms, s);
}

static cudaError_t dispatch_bwd(cgtp_plan p, const ConvBwdArgs& a, int sms, cudaStream_t s) {
  cudaError_t e = cudaErrorNotSupported;
#define CGTP_DBWD_ENTRY(A, B, C) \
  if (p->li == A && p->ls == B && p->lo == C) e = launch_conv_bwd<A, B, C>(a, sms, s);
  CGTP_CONFIGS(CGTP_DBWD_ENTRY)
  return e;
}

static int dd_slices(cgtp_plan p) {
  int s = 0;
#define CGTP_DD_SLICES_ENTRY(A, B, C) \
  if (p->li == A && p->ls == B && p->lo == C) s = conv_dd_slices<A, B, C>(p->mult);
  CGTP_CONFIGS(CGTP_DD_SLICES_ENTRY)
  return s;
}

// [E][NS] directional harmonics, then the harmonic-gradient partials: those
// of the first-order passes, or the fused pass's two sets, whichever is larger.
cgtp_status cgtp_conv_double_backward_workspace_size(cgtp_plan p, int n_edges, size_t* bytes) {
  if (!mode_is(p, CGTP_MODE_CONV_UVU) || n_edges < 0 || bytes == nullptr) return CGTP_ERR_INVALID_ARG;
  const size_t ns = (size_t)(p->ls + 1) * (p->ls + 1);
  const size_t u = (sizeof(float) * (size_t)n_edges * ns + 255) & ~(size_t)255;
  size_t bw = 0;
  cgtp_conv_backward_workspace_size(p, n_edges, &bw);
  const size_t dd = (sizeof(float) * 2 * (size_t)dd_slices(p) * (size_t)n_edges * ns + 255) & ~(size_t)255;
  *bytes = u + (dd > bw ? dd : bw);
  return CGTP_OK;
}

cgtp_status cgtp_conv_double_backward(cgtp_plan p, int n_nodes, int n_edges, const int* row_ptr, const int* col,
                                      const int* csc_ptr, const int* csc_edge, const int* csc_dst,
                                      const float* edge_vec, const float* x, const float* w, const float* grad_out,
                                      const float* gg_x, const float* gg_w, const float* gg_edge_vec, float* d_x,
                                      float* d_w, float* d_grad_out, float* d_edge_vec, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  if (!mode_is(p, CGTP_MODE_CONV_UVU) || n_nodes < 0 || n_edges < 0 || row_ptr == nullptr || csc_ptr == nullptr)
    return CGTP_ERR_INVALID_ARG;
  if (n_nodes > 0 && (x == nullptr || grad_out == nullptr)) return CGTP_ERR_INVALID_ARG;
  if (n_edges > 0 && (col == nullptr || csc_edge == nullptr || csc_dst == nullptr || edge_vec == nullptr ||
                      w == nullptr))
    return CGTP_ERR_INVALID_ARG;
  for (const void* q : {(const void*)x, (const void*)w, (const void*)grad_out, (const void*)gg_x, (const void*)gg_w,
                        (const void*)d_x, (const void*)d_w, (const void*)d_grad_out})
    if (!aligned16(q)) return CGTP_ERR_INVALID_ARG;
  const size_t ns = (size_t)(p->ls + 1) * (p->ls + 1);
  const size_t u_bytes = (sizeof(float) * (size_t)n_edges * ns + 255) & ~(size_t)255;
  const bool need_ws = n_edges > 0 && (gg_edge_vec != nullptr || d_edge_vec != nullptr);
  if (need_ws) {
    size_t need = 0;
    cgtp_conv_double_backward_workspace_size(p, n_edges, &need);
    if (workspace == nullptr || workspace_bytes < need || ((uintptr_t)workspace & 255u) != 0)
      return CGTP_ERR_WORKSPACE;
  }
  int sms = 0;
  cgtp_status st = ensure_device(&sms);
  if (st != CGTP_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (n_nodes == 0) return CGTP_OK;
  const size_t nx = (size_t)n_nodes * (p->li + 1) * (p->li + 1) * p->mult;
  const size_t ng = (size_t)n_nodes * (p->lo + 1) * (p->lo + 1) * p->mult;
  const size_t nw = (size_t)n_edges * p->n_paths * p->mult;
  cudaError_t e = cudaSuccess;
  auto zero = [&](float* q, size_t n) {
    if (q != nullptr && n > 0 && e == cudaSuccess) e = cudaMemsetAsync(q, 0, sizeof(float) * n, s);
  };
  if (n_edges == 0) {  // nothing depends on anything: every gradient is zero
    zero(d_x, nx);
    zero(d_grad_out, ng);
    return e == cudaSuccess ? CGTP_OK : cuda_fail(e);
  }
  float* uY = need_ws ? (float*)workspace : nullptr;                      // [E][NS] = (dY/dr) gg_edge_vec
  float* gsh = need_ws ? (float*)((char*)workspace + u_bytes) : nullptr;  // harmonic-gradient partials
  const bool gr = gg_edge_vec != nullptr;
  const int* abort_flag = nullptr;
  e = validate_graph(p, n_nodes, n_edges, row_ptr, col, edge_vec, csc_ptr, csc_edge, csc_dst, sms, s, &abort_flag);
  if (e != cudaSuccess) return cuda_fail(e);

  // Every cotangent given: the fused passes.  d grad_out by one forward that
  // reads W and gg_W once; d x, d W and the edge-vector term by one
  // source-centric pass that reads them once more and writes d W once.  The
  // two passes write disjoint outputs: the forward runs on a side lane,
  // forked from `s` and joined back, beside the (compute-heavier) source pass.
  if (gg_x != nullptr && gg_w != nullptr && gr) {
    const bool want_fwd = d_grad_out != nullptr;
    const bool want_bwd = d_x != nullptr || d_w != nullptr || d_edge_vec != nullptr;
    std::unique_lock<std::mutex> turn(side_lanes_mutex(kLanesDD), std::defer_lock);
    SideLanes* L = nullptr;
    cudaStream_t fs = s;
    if (want_fwd && want_bwd) {
      turn.lock();
      e = side_lanes(kLanesDD, &L);
      if (e == cudaSuccess) e = lanes_fork(L, 1, s);
      if (e != cudaSuccess) return cuda_fail(e);
      fs = L->side[0];
    }
    if (want_bwd) {
      ConvBwdArgs a{n_nodes, n_edges, csc_ptr, csc_edge, csc_dst, edge_vec, x, w, grad_out,
                    d_x, d_w, d_edge_vec, gsh, p->mult};
      a.abort_flag = abort_flag;
      a.x2 = gg_x;
      a.w2 = gg_w;
      a.gr_dir = gg_edge_vec;
      e = cudaErrorNotSupported;
#define CGTP_DDB_ENTRY(A, B, C) \
      if (p->li == A && p->ls == B && p->lo == C) e = launch_conv_dd_bwd<A, B, C>(a, sms, s);
      CGTP_CONFIGS(CGTP_DDB_ENTRY)
    }
    if (e == cudaSuccess && want_fwd) {
      ConvFwdArgs a{n_nodes, row_ptr, col, edge_vec, x, w, d_grad_out, p->mult};
      a.abort_flag = abort_flag;
      a.x2 = gg_x;
      a.w2 = gg_w;
      a.gr_dir = gg_edge_vec;
      e = cudaErrorNotSupported;
#define CGTP_DDF_ENTRY(A, B, C) \
      if (p->li == A && p->ls == B && p->lo == C) e = launch_conv_dd_fwd<A, B, C>(a, sms, fs);
      CGTP_CONFIGS(CGTP_DDF_ENTRY)
    }
    if (L != nullptr) {  // join even after an error, so the lane is not left forked
      const cudaError_t ej = lanes_join(L, 1, s);
      if (e == cudaSuccess) e = ej;
    }
    return e == cudaSuccess ? CGTP_OK : cuda_fail(e);
  }

  // Otherwise a sum of first-order passes with one argument replaced.
  if (gr) e = launch_sh_dir(p->ls, n_edges, edge_vec, gg_edge_vec, uY, sms, s);

  // d grad_out: forward convolutions with one argument replaced at a time
  //   (Y -> uY), (x -> gg_x), (W -> gg_w), summed
  if (d_grad_out != nullptr) {
    bool init = false;
    auto fwd = [&](const float* xx, const float* ww, const float* sh) {
      if (e != cudaSuccess) return;
      ConvFwdArgs a{n_nodes, row_ptr, col, edge_vec, xx, ww, d_grad_out, p->mult};
      a.abort_flag = abort_flag;
      a.sh = sh;
      a.accumulate = init ? 1 : 0;
      e = dispatch_fwd(p, a, sms, s);
      init = true;
    };
    if (gr) fwd(x, w, uY);
    if (gg_x) fwd(gg_x, w, nullptr);
    if (gg_w) fwd(x, gg_w, nullptr);
    if (!init) zero(d_grad_out, ng);
  }

  // d x and d W: backward convolutions, (Y -> uY) for both, then
  //   d x += grad_x with W -> gg_w and d W += grad_w with x -> gg_x (one launch)
  if (d_x != nullptr || d_w != nullptr) {
    bool init_x = false, init_w = false;
    if (gr && e == cudaSuccess) {
      ConvBwdArgs a{n_nodes, n_edges, csc_ptr, csc_edge, csc_dst, edge_vec, x, w, grad_out,
                    d_x, d_w, nullptr, nullptr, p->mult};
      a.abort_flag = abort_flag;
      a.sh = uY;
      e = dispatch_bwd(p, a, sms, s);
      init_x = d_x != nullptr;
      init_w = d_w != nullptr;
    }
    float* ox = gg_w ? d_x : nullptr;
    float* ow = gg_x ? d_w : nullptr;
    if ((ox != nullptr || ow != nullptr) && e == cudaSuccess) {
      // the two outputs accumulate together: both were written above or neither
      ConvBwdArgs a{n_nodes, n_edges, csc_ptr, csc_edge, csc_dst, edge_vec, gg_x ? gg_x : x, gg_w ? gg_w : w,
                    grad_out, ox, ow, nullptr, nullptr, p->mult};
      a.abort_flag = abort_flag;
      a.accumulate = gr ? 1 : 0;
      e = dispatch_bwd(p, a, sms, s);
      init_x = init_x || ox != nullptr;
      init_w = init_w || ow != nullptr;
    }
    if (!init_x) zero(d_x, nx);
    if (!init_w) zero(d_w, nw);
  }

  // d edge_vec: (dY/dr)^T of the harmonic gradients with x -> gg_x and with
  //   W -> gg_w, plus sum_b G_b (d2Y_b/dr2) gg_edge_vec with G the backward's own
  if (d_edge_vec != nullptr) {
    bool init = false;
    auto gy = [&](const float* xx, const float* ww, int mode_set, int mode_add) {
      if (e != cudaSuccess) return;
      ConvBwdArgs a{n_nodes, n_edges, csc_ptr, csc_edge, csc_dst, edge_vec, xx, ww, grad_out,
                    nullptr, nullptr, d_edge_vec, gsh, p->mult};
      a.abort_flag = abort_flag;
      a.gr_mode = init ? mode_add : mode_set;
      a.gr_dir = gg_edge_vec;
      e = dispatch_bwd_gy(p, a, sms, s);
      init = true;
    };
    if (gg_x) gy(gg_x, w, 0, 1);
    if (gg_w) gy(x, gg_w, 0, 1);
    if (gr) gy(x, w, 3, 2);
    if (!init) zero(d_edge_vec, (size_t)n_edges * 3);
  }
  return e == cudaSuccess ? CGTP_OK : cuda_fail(e);
}

// ---- fully connected (uvw) convolution ----
struct UvwLayout {
  int order[kMaxPaths];
  int count_l3[kLmaxTab + 1];
  size_t t_floats, packed_floats;
};
static bool uvw_layout(cgtp_plan p, int n_nodes, int mult_out, UvwLayout* L) {
  bool found = false;
#define CGTP_UVW_ORDER_ENTRY(A, B, C) \
  if (p->li == A && p->ls == B && p->lo == C) { conv_path_order<A, B, C>(L->order, L->count_l3); found = true; }
  CGTP_VARIANT_CONFIGS(CGTP_UVW_ORDER_ENTRY)
  if (!found) return false;
  L->t_floats = L->packed_floats = 0;
  for (int l3 = 0; l3 <= p->lo; ++l3) {
    L->t_floats += (size_t)n_nodes * (2 * l3 + 1) * L->count_l3[l3] * p->mult;
    L->packed_floats += (size_t)(2 * l3 + 1) * L->count_l3[l3] * p->mult * mult_out;
  }
  return true;
}
static size_t round256(size_t b) { return (b + 255) & ~(size_t)255; }

cgtp_status cgtp_uvw_forward_workspace_size(cgtp_plan p, int n_nodes, int mult_out, size_t* bytes) {
  if (!mode_is(p, CGTP_MODE_CONV_UVW) || n_nodes < 0 || mult_out <= 0 || bytes == nullptr)
    return CGTP_ERR_INVALID_ARG;
  UvwLayout L;
  if (!uvw_layout(p, n_nodes, mult_out, &L)) return CGTP_ERR_UNSUPPORTED;
  *bytes = round256(sizeof(float) * L.t_floats) + round256(sizeof(float) * L.packed_floats) +
           uvw_gemm_workspace(n_nodes, p->lo, L.count_l3, p->mult, mult_out);
  return CGTP_OK;
}

cgtp_status cgtp_uvw_forward(cgtp_plan p, int n_nodes, int n_edges, const int* row_ptr, const int* col,
                             const float* edge_vec, const float* x, const float* w, const float* mix, int mult_out,
                             float* out, void* workspace, size_t workspace_bytes, void* stream) {
  if (!mode_is(p, CGTP_MODE_CONV_UVW) || n_nodes < 0 || n_edges < 0 || row_ptr == nullptr || mult_out <= 0 ||
      mix == nullptr)
    return CGTP_ERR_INVALID_ARG;
  if (n_nodes > 0 && (x == nullptr || out == nullptr)) return CGTP_ERR_INVALID_ARG;
  if (n_edges > 0 && (col == nullptr || edge_vec == nullptr || w == nullptr)) return CGTP_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(out)) return CGTP_ERR_INVALID_ARG;
  if (p->mult % 4 != 0 || mult_out % 4 != 0) return CGTP_ERR_UNSUPPORTED;  // 16-byte GEMM rows
  if (n_nodes == 0) return CGTP_OK;
  size_t need = 0;
  cgtp_status st = cgtp_uvw_forward_workspace_size(p, n_nodes, mult_out, &need);
  if (st != CGTP_OK) return st;
  if (workspace == nullptr || workspace_bytes < need || ((uintptr_t)workspace & 255u) != 0)
    return CGTP_ERR_WORKSPACE;
  int sms = 0;
  st = ensure_device(&sms);
  if (st != CGTP_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  UvwLayout L;
  uvw_layout(p, n_nodes, mult_out, &L);
  float* t = (float*)workspace;
  float* packed = (float*)((char*)workspace + round256(sizeof(float) * L.t_floats));
  void* gws = (char*)packed + round256(sizeof(float) * L.packed_floats);
  const size_t gws_bytes = workspace_bytes - round256(sizeof(float) * L.t_floats) -
                           round256(sizeof(float) * L.packed_floats);
  // Per l3 block, on the block's lane: stage 1, the per-path messages t of the
  // block's paths (channelwise convolution, paths kept apart); the block's
  // packed mixing matrices; stage 2, the block's mixing GEMM (tensor cores).
  // The blocks' lanes overlap, so one block's GEMM runs beside the next
  // block's messages.  Output blocks that no path reaches are zero.
  ConvFwdArgs a{n_nodes, row_ptr, col, edge_vec, x, w, t, p->mult};
  cudaError_t e = validate_graph(p, n_nodes, n_edges, row_ptr, col, edge_vec, nullptr, nullptr, nullptr, sms, s,
                                 &a.abort_flag);
  if (e != cudaSuccess) return cuda_fail(e);
  for (int l3 = 0; l3 <= p->lo && e == cudaSuccess; ++l3)
    if (L.count_l3[l3] == 0) {
      const int no = (p->lo + 1) * (p->lo + 1);
      e = cudaMemset2DAsync(out + (size_t)l3 * l3 * mult_out, sizeof(float) * no * mult_out, 0,
                            sizeof(float) * (2 * l3 + 1) * mult_out, n_nodes, s);
    }
  auto stage1 = [&](int l3, cudaStream_t st) -> cudaError_t {
    if (L.count_l3[l3] == 0) return cudaSuccess;
    cudaError_t r = cudaErrorNotSupported;
#define CGTP_UVW_PATHS_ENTRY(A, B, C) \
    if (p->li == A && p->ls == B && p->lo == C) r = launch_conv_paths<A, B, C>(a, sms, st, l3);
    CGTP_VARIANT_CONFIGS(CGTP_UVW_PATHS_ENTRY)
    if (r == cudaSuccess)
      r = launch_uvw_pack_l3(p->n_paths, p->mult, mult_out, p->lo, L.order, L.count_l3, mix, packed, l3, st);
    return r;
  };
  if (e == cudaSuccess)
    e = launch_uvw_gemm_after(n_nodes, p->lo, L.count_l3, p->mult, mult_out, t, packed, out, gws, gws_bytes, s,
                              stage1);
  if (e == cudaErrorNotSupported) return CGTP_ERR_UNSUPPORTED;
  return e == cudaSuccess ? CGTP_OK : cuda_fail(e);
}

struct UvwBwdParts {
  size_t gt, t, packed, part, gemm, bwd;  // bytes of each workspace part
};
static bool uvw_bwd_parts(cgtp_plan p, int n_nodes, int n_edges, int mult_out, bool want_mix, bool want_r,
                          UvwLayout* L, UvwBwdParts* W) {
  if (!uvw_layout(p, n_nodes, mult_out, L)) return false;
  size_t part = 0;
  for (int l3 = 0; l3 <= p->lo; ++l3) part += (size_t)(2 * l3 + 1) * L->count_l3[l3] * p->mult * mult_out;
  W->gt = round256(sizeof(float) * L->t_floats);
  W->t = want_mix ? W->gt : 0;
  W->packed = round256(sizeof(float) * L->packed_floats);
  W->part = want_mix ? round256(sizeof(float) * part) : 0;
  W->gemm = uvw_bwd_gemm_workspace(n_nodes, p->lo, L->count_l3, p->mult, mult_out);
  size_t bw = 0;
  if (want_r) cgtp_conv_backward_workspace_size(p, n_edges, &bw);
  W->bwd = bw;
  return true;
}

cgtp_status cgtp_uvw_backward_workspace_size(cgtp_plan p, int n_nodes, int n_edges, int mult_out, size_t* bytes) {
  if (!mode_is(p, CGTP_MODE_CONV_UVW) || n_nodes < 0 || n_edges < 0 || mult_out <= 0 || bytes == nullptr)
    return CGTP_ERR_INVALID_ARG;
  UvwLayout L;
  UvwBwdParts W;
  if (!uvw_bwd_parts(p, n_nodes, n_edges, mult_out, true, true, &L, &W)) return CGTP_ERR_UNSUPPORTED;
  *bytes = W.gt + W.t + W.packed + W.part + W.gemm + W.bwd;
  return CGTP_OK;
}

cgtp_status cgtp_uvw_backward(cgtp_plan p, int n_nodes, int n_edges, const int* row_ptr, const int* col,
                              const int* csc_ptr, const int* csc_edge, const int* csc_dst, const float* edge_vec,
                              const float* x, const float* w, const float* mix, int mult_out, const float* grad_out,
                              float* grad_x, float* grad_w, float* grad_mix, float* grad_edge_vec, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (!mode_is(p, CGTP_MODE_CONV_UVW) || n_nodes < 0 || n_edges < 0 || row_ptr == nullptr || csc_ptr == nullptr ||
      mult_out <= 0 || mix == nullptr)
    return CGTP_ERR_INVALID_ARG;
  if (n_nodes > 0 && (x == nullptr || grad_out == nullptr)) return CGTP_ERR_INVALID_ARG;
  if (n_edges > 0 && (col == nullptr || csc_edge == nullptr || csc_dst == nullptr || edge_vec == nullptr ||
                      w == nullptr))
    return CGTP_ERR_INVALID_ARG;
  for (const void* q : {(const void*)x, (const void*)w, (const void*)mix, (const void*)grad_out, (const void*)grad_x,
                        (const void*)grad_w, (const void*)grad_mix})
    if (!aligned16(q)) return CGTP_ERR_INVALID_ARG;
  if (p->mult % 4 != 0 || mult_out % 4 != 0) return CGTP_ERR_UNSUPPORTED;
  if (n_nodes == 0) return CGTP_OK;
  UvwLayout L;
  UvwBwdParts W;
  if (!uvw_bwd_parts(p, n_nodes, n_edges, mult_out, grad_mix != nullptr, grad_edge_vec != nullptr, &L, &W))
    return CGTP_ERR_UNSUPPORTED;
  const size_t need = W.gt + W.t + W.packed + W.part + W.gemm + W.bwd;
  if (workspace == nullptr || workspace_bytes < need || ((uintptr_t)workspace & 255u) != 0)
    return CGTP_ERR_WORKSPACE;
  int sms = 0;
  cgtp_status st = ensure_device(&sms);
  if (st != CGTP_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  char* ws = (char*)workspace;
  float* gt = (float*)ws;
  float* t = (float*)(ws + W.gt);
  float* packed_t = (float*)(ws + W.gt + W.t);
  float* part = (float*)(ws + W.gt + W.t + W.packed);
  void* gws = ws + W.gt + W.t + W.packed + W.part;
  float* bws = (float*)(ws + W.gt + W.t + W.packed + W.part + W.gemm);
  const int* abort_flag = nullptr;
  cudaError_t e = validate_graph(p, n_nodes, n_edges, row_ptr, col, edge_vec, csc_ptr, csc_edge, csc_dst, sms, s,
                                 &abort_flag);
  if (e != cudaSuccess) return cuda_fail(e);
  // per-path output gradients gt (tensor cores)
  e = launch_uvw_pack_t(p->n_paths, p->mult, mult_out, p->lo, L.order, L.count_l3, mix, packed_t, s);
  if (e == cudaSuccess)
    e = launch_uvw_gt(n_nodes, p->lo, L.count_l3, p->mult, mult_out, grad_out, packed_t, gt, gws, W.gemm, s);
  // channelwise backward with one output gradient per path
  if (e == cudaSuccess && (grad_x != nullptr || grad_w != nullptr || grad_edge_vec != nullptr)) {
    if (n_edges == 0) {
      if (grad_x) e = cudaMemsetAsync(grad_x, 0, sizeof(float) * (size_t)n_nodes * (p->li + 1) * (p->li + 1) * p->mult, s);
    } else {
      ConvBwdArgs a{n_nodes, n_edges, csc_ptr, csc_edge, csc_dst, edge_vec, x, w, gt,
                    grad_x, grad_w, grad_edge_vec, bws, p->mult};
      a.abort_flag = abort_flag;
      e = cudaErrorNotSupported;
#define CGTP_UVWB_BWD_ENTRY(A, B, C) \
      if (p->li == A && p->ls == B && p->lo == C) e = launch_conv_bwd_paths<A, B, C>(a, sms, s);
      CGTP_VARIANT_CONFIGS(CGTP_UVWB_BWD_ENTRY)
    }
  }
  // grad_mix from the recomputed per-path messages t (tensor cores)
  if (e == cudaSuccess && grad_mix != nullptr) {
    ConvFwdArgs a{n_nodes, row_ptr, col, edge_vec, x, w, t, p->mult};
    a.abort_flag = abort_flag;
    e = cudaErrorNotSupported;
#define CGTP_UVWB_PATHS_ENTRY(A, B, C) \
    if (p->li == A && p->ls == B && p->lo == C) e = launch_conv_paths<A, B, C>(a, sms, s);
    CGTP_VARIANT_CONFIGS(CGTP_UVWB_PATHS_ENTRY)
    if (e == cudaSuccess)
      e = launch_uvw_grad_mix(n_nodes, p->n_paths, p->lo, L.order, L.count_l3, p->mult, mult_out, t, grad_out, part,
                              grad_mix, gws, W.gemm, s);
  }
  if (e == cudaErrorNotSupported) return CGTP_ERR_UNSUPPORTED;
  return e == cudaSuccess ? CGTP_OK : cuda_fail(e);
}

cgtp_status cgtp_forces(int n_nodes, int n_edges, const int* row_ptr, const int* csc_ptr, const int* csc_edge,
                        const float* grad_edge_vec, float* forces, void* stream) {
  if (n_nodes < 0 || n_edges < 0 || row_ptr == nullptr || csc_ptr == nullptr) return CGTP_ERR_INVALID_ARG;
  if (n_nodes > 0 && forces == nullptr) return CGTP_ERR_INVALID_ARG;
  if (n_edges > 0 && (csc_edge == nullptr || grad_edge_vec == nullptr)) return CGTP_ERR_INVALID_ARG;
  int sms = 0;
  cgtp_status st = ensure_device(&sms);
  if (st != CGTP_OK) return st;
  cudaError_t e = launch_forces(n_nodes, row_ptr, csc_ptr, csc_edge, grad_edge_vec, forces, sms, (cudaStream_t)stream);
  return e == cudaSuccess ? CGTP_OK : cuda_fail(e);
}

// Weights per edge of a convolution plan: one row per path, or one shared row.
static int edge_weights(cgtp_plan p) { return p->mode == CGTP_MODE_CONV_UVU_SHARED ? p->mult : p->n_paths * p->mult; }

cgtp_status cgtp_gather_rows(int n, int row_floats, const int* idx, const float* src, float* dst, void* stream) {
  if (n < 0 || row_floats < 0) return CGTP_ERR_INVALID_ARG;
  if (n > 0 && row_floats > 0 && (idx == nullptr || src == nullptr || dst == nullptr)) return CGTP_ERR_INVALID_ARG;
  int sms = 0;
  cgtp_status st = ensure_device(&sms);
  if (st != CGTP_OK) return st;
  cudaError_t e = launch_rows(false, n, row_floats, idx, src, dst, sms, (cudaStream_t)stream);
  return e == cudaSuccess ? CGTP_OK : cuda_fail(e);
}

cgtp_status cgtp_scatter_add_rows(int n, int row_floats, const int* idx, const float* src, float* dst,
                                  void* stream) {
  if (n < 0 || row_floats < 0) return CGTP_ERR_INVALID_ARG;
  if (n > 0 && row_floats > 0 && (idx == nullptr || src == nullptr || dst == nullptr)) return CGTP_ERR_INVALID_ARG;
  int sms = 0;
  cgtp_status st = ensure_device(&sms);
  if (st != CGTP_OK) return st;
  cudaError_t e = launch_rows(true, n, row_floats, idx, src, dst, sms, (cudaStream_t)stream);
  return e == cudaSuccess ? CGTP_OK : cuda_fail(e);
}

cgtp_status cgtp_radial_forward(cgtp_plan p, int n_edges, const float* edge_vec, float rc, const float* W1,
                                const float* W2, float* w, void* stream) {
  if (p == nullptr || p->mode == CGTP_MODE_PAIR_UVU || n_edges < 0 || !(rc > 0.f)) return CGTP_ERR_INVALID_ARG;
  if (n_edges > 0 && (edge_vec == nullptr || W1 == nullptr || W2 == nullptr || w == nullptr))
    return CGTP_ERR_INVALID_ARG;
  if (!aligned16(W2) || !aligned16(w)) return CGTP_ERR_INVALID_ARG;
  int sms = 0;
  cgtp_status st = ensure_device(&sms);
  if (st != CGTP_OK) return st;
  cudaError_t e =
      launch_radial_fwd(n_edges, edge_weights(p), edge_vec, rc, W1, W2, w, sms, (cudaStream_t)stream);
  return e == cudaSuccess ? CGTP_OK : cuda_fail(e);
}

cgtp_status cgtp_radial_backward(cgtp_plan p, int n_edges, const float* edge_vec, float rc, const float* W1,
                                 const float* W2, const float* grad_w, float* grad_edge_vec, void* stream) {
  if (p == nullptr || p->mode == CGTP_MODE_PAIR_UVU || n_edges < 0 || !(rc > 0.f)) return CGTP_ERR_INVALID_ARG;
  if (n_edges > 0 && (edge_vec == nullptr || W1 == nullptr || W2 == nullptr || grad_w == nullptr ||
                      grad_edge_vec == nullptr))
    return CGTP_ERR_INVALID_ARG;
  if (!aligned16(W2) || !aligned16(grad_w)) return CGTP_ERR_INVALID_ARG;
  int sms = 0;
  cgtp_status st = ensure_device(&sms);
  if (st != CGTP_OK) return st;
  cudaError_t e = launch_radial_bwd(n_edges, edge_weights(p), edge_vec, rc, W1, W2, grad_w, grad_edge_vec, sms,
                                    (cudaStream_t)stream);
  return e == cudaSuccess ? CGTP_OK : cuda_fail(e);
}

cgtp_status cgtp_tp_forward(cgtp_plan p, int batch, const float* x, const float* y, const float* w, float* z,
                            void* stream) {
  if (!mode_is(p, CGTP_MODE_PAIR_UVU) || batch < 0) return CGTP_ERR_INVALID_ARG;
  if (batch > 0 && (x == nullptr || y == nullptr || w == nullptr || z == nullptr)) return CGTP_ERR_INVALID_ARG;
  int sms = 0;
  cgtp_status st = ensure_device(&sms);
  if (st != CGTP_OK) return st;
  TPArgs a{batch, x, y, w, nullptr, z, nullptr, nullptr, nullptr, nullptr, p->mult};
  cudaError_t e = cudaErrorNotSupported;
#define CGTP_TPF_ENTRY(A, B, C) \
  if (p->li == A && p->ls == B && p->lo == C) e = launch_tp_fwd<A, B, C>(a, sms, (cudaStream_t)stream);
  CGTP_CONFIGS(CGTP_TPF_ENTRY)
  return e == cudaSuccess ? CGTP_OK : cuda_fail(e);
}

cgtp_status cgtp_tp_backward_workspace_size(cgtp_plan p, int batch, size_t* bytes) {
  if (!mode_is(p, CGTP_MODE_PAIR_UVU) || batch < 0 || bytes == nullptr) return CGTP_ERR_INVALID_ARG;
  const size_t b = sizeof(float) * (size_t)tp_chunks(batch) * p->n_paths * p->mult;
  *bytes = (b + 255) & ~(size_t)255;
  return CGTP_OK;
}

cgtp_status cgtp_tp_backward(cgtp_plan p, int batch, const float* x, const float* y, const float* w,
                             const float* grad_z, float* grad_x, float* grad_y, float* grad_w, void* workspace,
                             size_t workspace_bytes, void* stream) {
  if (!mode_is(p, CGTP_MODE_PAIR_UVU) || batch < 0) return CGTP_ERR_INVALID_ARG;
  if (batch > 0 && (x == nullptr || y == nullptr || w == nullptr || grad_z == nullptr)) return CGTP_ERR_INVALID_ARG;
  if (grad_w != nullptr) {
    size_t need = 0;
    cgtp_tp_backward_workspace_size(p, batch, &need);
    if (workspace == nullptr || workspace_bytes < need) return CGTP_ERR_WORKSPACE;
  }
  int sms = 0;
  cgtp_status st = ensure_device(&sms);
  if (st != CGTP_OK) return st;
  TPArgs a{batch, x, y, w, grad_z, nullptr, grad_x, grad_y, grad_w, grad_w ? (float*)workspace : nullptr, p->mult};
  cudaError_t e = cudaErrorNotSupported;
#define CGTP_TPB_ENTRY(A, B, C) \
  if (p->li == A && p->ls == B && p->lo == C) e = launch_tp_bwd<A, B, C>(a, sms, (cudaStream_t)stream);
  CGTP_CONFIGS(CGTP_TPB_ENTRY)
  return e == cudaSuccess ? CGTP_OK : cuda_fail(e);
}

static size_t cp_device_smem_limit() {
  int dev = 0, v = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return 0;
  return (size_t)v;
}

static size_t cp_smem_for(cgtp_plan p, int rank, bool factor_grads) {
  size_t b = 0;
#define CGTP_CPS_ENTRY(A, B, C) \
  if (p->li == A && p->ls == B && p->lo == C) b = cp_smem_bytes<A, B, C>(rank, factor_grads);
  CGTP_CONFIGS(CGTP_CPS_ENTRY)
  return b;
}

cgtp_status cgtp_cp_forward(cgtp_plan p, int rank, int batch, const float* A, const float* B, const float* C,
                            const float* x, const float* y, float* z, void* stream) {
  if (!mode_is(p, CGTP_MODE_PAIR_UVU) || rank < 1 || batch < 0) return CGTP_ERR_INVALID_ARG;
  if (A == nullptr || B == nullptr || C == nullptr) return CGTP_ERR_INVALID_ARG;
  if (batch > 0 && (x == nullptr || y == nullptr || z == nullptr)) return CGTP_ERR_INVALID_ARG;
  int sms = 0;
  cgtp_status st = ensure_device(&sms);
  if (st != CGTP_OK) return st;
  const size_t need = cp_smem_for(p, rank, false);
  if (need == 0 || need > cp_device_smem_limit()) return CGTP_ERR_UNSUPPORTED;
  CPArgs a{batch, p->mult, rank, A, B, C, x, y, nullptr, z, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
  cudaError_t e = cudaErrorNotSupported;
#define CGTP_CPF_ENTRY(LA, LB, LC) \
  if (p->li == LA && p->ls == LB && p->lo == LC) e = launch_cp_fwd<LA, LB, LC>(a, (cudaStream_t)stream);
  CGTP_CONFIGS(CGTP_CPF_ENTRY)
  return e == cudaSuccess ? CGTP_OK : cuda_fail(e);
}

cgtp_status cgtp_cp_backward_workspace_size(cgtp_plan p, int rank, int batch, size_t* bytes) {
  if (!mode_is(p, CGTP_MODE_PAIR_UVU) || rank < 1 || batch < 0 || bytes == nullptr) return CGTP_ERR_INVALID_ARG;
  const int d1 = (p->li + 1) * (p->li + 1), d2 = (p->ls + 1) * (p->ls + 1), d3 = (p->lo + 1) * (p->lo + 1);
  const size_t b = sizeof(float) * (size_t)cp_bwd_blocks(batch, p->mult) * (size_t)(d1 + d2 + d3) * (size_t)rank;
  *bytes = (b + 255) & ~(size_t)255;
  return CGTP_OK;
}

cgtp_status cgtp_cp_backward(cgtp_plan p, int rank, int batch, const float* A, const float* B, const float* C,
                             const float* x, const float* y, const float* grad_z, float* grad_x, float* grad_y,
                             float* grad_A, float* grad_B, float* grad_C, void* workspace, size_t workspace_bytes,
                             void* stream) {
  if (!mode_is(p, CGTP_MODE_PAIR_UVU) || rank < 1 || batch < 0) return CGTP_ERR_INVALID_ARG;
  if (A == nullptr || B == nullptr || C == nullptr) return CGTP_ERR_INVALID_ARG;
  if (batch > 0 && (x == nullptr || y == nullptr || grad_z == nullptr)) return CGTP_ERR_INVALID_ARG;
  const bool gf = grad_A != nullptr || grad_B != nullptr || grad_C != nullptr;
  if (gf && batch > 0) {
    size_t need = 0;
    cgtp_cp_backward_workspace_size(p, rank, batch, &need);
    if (workspace == nullptr || workspace_bytes < need) return CGTP_ERR_WORKSPACE;
  }
  int sms = 0;
  cgtp_status st = ensure_device(&sms);
  if (st != CGTP_OK) return st;
  const size_t need = cp_smem_for(p, rank, gf);
  if (need == 0 || need > cp_device_smem_limit()) return CGTP_ERR_UNSUPPORTED;
  CPArgs a{batch, p->mult, rank, A, B, C, x, y, grad_z, nullptr, grad_x, grad_y, grad_A, grad_B, grad_C,
           gf ? (float*)workspace : nullptr};
  cudaError_t e = cudaErrorNotSupported;
#define CGTP_CPB_ENTRY(LA, LB, LC) \
  if (p->li == LA && p->ls == LB && p->lo == LC) e = launch_cp_bwd<LA, LB, LC>(a, (cudaStream_t)stream);
  CGTP_CONFIGS(CGTP_CPB_ENTRY)
  return e == cudaSuccess ? CGTP_OK : cuda_fail(e);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free variant of the edge-free tensor-product backward.
//
// Some callers cannot allocate device memory when they call this library:
// a host framework that owns all device memory through its own allocator and
// forbids direct cudaMalloc, or a time-stepping loop (molecular dynamics)
// that must not allocate after set-up because an allocation can stall the
// device or fail part-way through a run.  cgtp_tp_backward needs a caller
// workspace for its per-chunk grad_w partial sums; this variant keeps them
// instead in the fixed array below, which every GPU that loads the library
// holds until the process exits.
namespace cgtp {
namespace {

// 2 MiB: tp_chunks(batch) * n_paths * mult floats must fit (at most 64
// chunks, so n_paths * mult <= 8192, e.g. 34 paths x 128 channels at l = 3).
constexpr size_t kTpNoAllocFloats = size_t(1) << 19;
static __device__ __align__(256) float g_tp_noalloc_scratch[kTpNoAllocFloats];

std::mutex g_noalloc_mutex;
std::vector<float*> g_noalloc_ptr;  // device address of the array, per device (nullptr until looked up)

// The array's name in host code is only a host-side stand-in; the device
// address is looked up once per device, with that device current.
cgtp_status noalloc_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if ((int)g_noalloc_ptr.size() <= dev) g_noalloc_ptr.resize(dev + 1, nullptr);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_tp_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    g_noalloc_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return CGTP_OK;
}

}  // namespace
}  // namespace cgtp

extern "C" cgtp_status cgtp_tp_backward_noalloc(cgtp_plan p, int batch, const float* x, const float* y,
                                                const float* w, const float* grad_z, float* grad_x,
                                                float* grad_y, float* grad_w, void* stream) {
  if (!mode_is(p, CGTP_MODE_PAIR_UVU) || batch < 0) return CGTP_ERR_INVALID_ARG;
  if (batch > 0 && (x == nullptr || y == nullptr || w == nullptr || grad_z == nullptr)) return CGTP_ERR_INVALID_ARG;
  float* scratch = nullptr;
  if (grad_w != nullptr) {
    const size_t need = (size_t)tp_chunks(batch) * p->n_paths * p->mult;
    if (need > kTpNoAllocFloats) return CGTP_ERR_WORKSPACE;  // beyond the built-in scratch
  }
  int sms = 0;
  cgtp_status st = ensure_device(&sms);
  if (st != CGTP_OK) return st;
  if (grad_w != nullptr) {
    st = noalloc_scratch(&scratch);
    if (st != CGTP_OK) return st;
  }
  TPArgs a{batch, x, y, w, grad_z, nullptr, grad_x, grad_y, grad_w, scratch, p->mult};
  cudaError_t e = cudaErrorNotSupported;
#define CGTP_TPB_NOALLOC_ENTRY(A, B, C) \
  if (p->li == A && p->ls == B && p->lo == C) e = launch_tp_bwd<A, B, C>(a, sms, (cudaStream_t)stream);
  CGTP_CONFIGS(CGTP_TPB_NOALLOC_ENTRY)
  return e == cudaSuccess ? CGTP_OK : cuda_fail(e);
}
