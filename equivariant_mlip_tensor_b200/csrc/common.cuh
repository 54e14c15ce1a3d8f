// Device-side helpers shared by the kernels: compile-time loops, the
// constant-memory coefficient tables, cache-hinted vector loads and the
// launch-argument structs.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <type_traits>
#include <utility>

#include "structure.h"

namespace cgtp {

// ---- compile-time loop: f(std::integral_constant<int, I>) for I in [B, E) ----
template <int B, class F, int... Is>
__device__ __forceinline__ void static_for_impl(F&& f, std::integer_sequence<int, Is...>) {
  (f(std::integral_constant<int, B + Is>{}), ...);
}
template <int B, int E, class F>
__device__ __forceinline__ void static_for(F&& f) {
  if constexpr (E > B) static_for_impl<B>(f, std::make_integer_sequence<int, E - B>{});
}
template <int B, class F, int... Is>
void static_for_host_impl(F&& f, std::integer_sequence<int, Is...>) {
  (f(std::integral_constant<int, B + Is>{}), ...);
}
template <int B, int E, class F>
void static_for_host(F&& f) {
  if constexpr (E > B) static_for_host_impl<B>(f, std::make_integer_sequence<int, E - B>{});
}

// ---- coefficient tables.  Every translation unit that needs them holds its
// own constant-memory copy and registers an uploader at load time; plan
// creation runs every registered uploader once per device. ----
using UploadFn = cudaError_t (*)(const float* cg, const float* shk);
int register_table_uploader(UploadFn fn);  // host, defined in abi.cu

#define CGTP_DEFINE_CONSTANT_TABLES()                                              \
  static __constant__ float c_cg[kTableSize];                                      \
  static __constant__ float c_shk[kShkSize];                                       \
  static cudaError_t upload_tables_here(const float* cg, const float* shk) {       \
    cudaError_t e = cudaMemcpyToSymbol(c_cg, cg, sizeof(float) * kTableSize);      \
    if (e != cudaSuccess) return e;                                                \
    return cudaMemcpyToSymbol(c_shk, shk, sizeof(float) * kShkSize);               \
  }                                                                                \
  static const int tables_registered_here = register_table_uploader(&upload_tables_here);

// ---- programmatic dependent launch (sm_90 and later) ----
// A grid launched with programmatic stream serialization may start once every
// block of the grid before it has called grid_dependents_launch() (or
// exited); grid_dependency_wait() then blocks until that preceding grid has
// completed and its writes are visible.  Both are no-ops for a grid launched
// in plain stream order.
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Host: launch kern<<<grid, block, smem, stream>>>(args...), with programmatic
// stream serialization when pdl is set.
template <class... P, class... A>
cudaError_t launch_kernel(void (*kern)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, bool pdl,
                          A&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...);
}

// ---- loads / stores with cache hints ----
__device__ __forceinline__ float4 ld_stream(const float* p) {  // read once: evict first
  return __ldcs(reinterpret_cast<const float4*>(p));
}
__device__ __forceinline__ float4 ld_ro(const float* p) {  // read-only, reused: cached
  return __ldg(reinterpret_cast<const float4*>(p));
}
__device__ __forceinline__ void st_stream(float* p, float4 v) {
  __stcs(reinterpret_cast<float4*>(p), v);
}
__device__ __forceinline__ void st_f4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }

// Bulk prefetch of [p, p + bytes) into L2 (one TMA instruction; p and bytes
// multiples of 16).
__device__ __forceinline__ void prefetch_l2(const void* p, unsigned bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ void f4_to(float (&a)[4], float4 v) {
  a[0] = v.x; a[1] = v.y; a[2] = v.z; a[3] = v.w;
}
__device__ __forceinline__ float4 to_f4(const float (&a)[4]) { return make_float4(a[0], a[1], a[2], a[3]); }

// Bits of the graph validation (graph.cu) that make a launch unsafe (offsets
// and indices out of range): a kernel given a flag word with any of them set
// does no work.
constexpr int kGraphUnsafeBits = 1 | 2 | 16 | 32;

// ---- launch arguments ----
struct ConvFwdArgs {
  int n_nodes;
  const int* row_ptr;
  const int* col;
  const float* edge_vec;
  const float* x;
  const float* w;
  float* out;
  int mult;
  // optional: per-edge harmonics [n_edges][(L_sh+1)^2] used instead of
  // Y(edge_vec) (the double backward substitutes directional derivatives)
  const float* sh = nullptr;
  int accumulate = 0;  // add onto out instead of overwriting it
  // checked mode: the plan's validation flags, written by a validation
  // launch earlier in the stream; the kernel does nothing if they are unsafe
  const int* abort_flag = nullptr;
  // the double backward's fused forward: out = conv(x2, w, Y) + conv(x, w2, Y)
  // + conv(x, w, (dY/dr) gr_dir)
  const float* x2 = nullptr;
  const float* w2 = nullptr;
  const float* gr_dir = nullptr;
};

struct ConvBwdArgs {
  int n_nodes;
  int n_edges;
  const int* csc_ptr;
  const int* csc_edge;
  const int* csc_dst;
  const float* edge_vec;
  const float* x;
  const float* w;
  const float* grad_out;
  float* grad_x;
  float* grad_w;
  float* grad_edge_vec;
  float* grad_sh;   // workspace [slices][n_edges][NS]
  int mult;
  const float* sh = nullptr;  // optional per-edge harmonics replacing Y(edge_vec)
  int accumulate = 0;         // add onto grad_x and grad_w instead of overwriting them
  // grad_edge_vec from the harmonic gradient G (summed over the slices):
  // 0: = (dY/dr)^T G, 1: += (dY/dr)^T G, 2: += sum_b G_b (d2Y_b/dr2) gr_dir,
  // 3: = sum_b G_b (d2Y_b/dr2) gr_dir
  int gr_mode = 0;
  const float* gr_dir = nullptr;  // [n_edges][3], for gr_mode 2 and 3
  const int* abort_flag = nullptr;  // checked mode, as in ConvFwdArgs
  // the double backward's fused pass: second features and weights (the
  // cotangents gg_x, gg_w); gr_dir is then the cotangent gg_r
  const float* x2 = nullptr;
  const float* w2 = nullptr;
};

struct TPArgs {
  int batch;
  const float* x;
  const float* y;
  const float* w;
  const float* grad_z;  // bwd
  float* z;             // fwd
  float* grad_x;
  float* grad_y;
  float* grad_w;
  float* partial;       // workspace [chunks][P][mult]
  int mult;
};

// Edge-free tensor product: batch rows per block and the number of batch
// chunks whose grad_w partials the backward keeps in its workspace.
constexpr int kTpRows = 8;
constexpr int kTpChunksMax = 64;
inline int tp_chunks(int batch) {
  int ch = (batch + kTpRows - 1) / kTpRows;
  if (ch > kTpChunksMax) ch = kTpChunksMax;
  return ch < 1 ? 1 : ch;
}

}  // namespace cgtp
