// Host-side launchers of every kernel family (defined in the .cu files; the
// per-shape ones are instantiated once per entry of configs.h).
#pragma once

#include <cuda_runtime.h>

#include <functional>
#include <mutex>

#include "common.cuh"

namespace cgtp {

// ---- side streams (lanes.cu) ----
// Launches of one call that write disjoint outputs run on lanes forked from
// the caller's stream (lanes_fork: lanes 0..n-1 wait for it) and joined back
// (lanes_join: the caller's stream waits for them).  A host thread holds
// side_lanes_mutex(pool) from the fork to the join (the events are shared).
constexpr int kMaxSideLanes = 4;
enum { kLanesBwd = 0, kLanesUvw = 1, kLanesDD = 2, kLanePools = 3 };
struct SideLanes {
  cudaStream_t side[kMaxSideLanes];
  cudaEvent_t fork, join[kMaxSideLanes];
};
cudaError_t side_lanes(int pool, SideLanes** out);
std::mutex& side_lanes_mutex(int pool);
cudaError_t lanes_fork(SideLanes* L, int n, cudaStream_t s);
cudaError_t lanes_join(SideLanes* L, int n, cudaStream_t s);

// Arguments of the CP-decomposed tensor product (cp.cu): factors A [d3][R],
// B [d1][R], C [d2][R]; features [batch][d][mult]; partial: the backward's
// per-block factor-gradient partials (cp_bwd_blocks x (d1 + d2 + d3) x R floats).
struct CPArgs {
  int batch, mult, rank;
  const float *A, *B, *C, *x, *y, *grad_z;
  float *z, *grad_x, *grad_y, *grad_A, *grad_B, *grad_C, *partial;
};
// The backward with factor gradients walks (pair, channel) items in tiles of
// 64; each block takes cp_bwd_tiles_per_block consecutive tiles (at most 512
// blocks), a fixed function of the problem size, so the partials and their
// summation order do not depend on the device.
constexpr int kCpItemsPerTile = 64;
constexpr long long kCpMaxPartials = 512;
inline long long cp_bwd_tiles(int batch, int mult) {
  return ((long long)batch * mult + kCpItemsPerTile - 1) / kCpItemsPerTile;
}
inline long long cp_bwd_tiles_per_block(int batch, int mult) {
  const long long t = cp_bwd_tiles(batch, mult);
  return t <= kCpMaxPartials ? 1 : (t + kCpMaxPartials - 1) / kCpMaxPartials;
}
inline long long cp_bwd_blocks(int batch, int mult) {
  const long long tpb = cp_bwd_tiles_per_block(batch, mult);
  return (cp_bwd_tiles(batch, mult) + tpb - 1) / tpb;
}
template <int LI, int LS, int LO>
size_t cp_smem_bytes(int rank, bool factor_grads);
template <int LI, int LS, int LO>
cudaError_t launch_cp_fwd(const CPArgs& a, cudaStream_t stream);
template <int LI, int LS, int LO>
cudaError_t launch_cp_bwd(const CPArgs& a, cudaStream_t stream);

template <int LI, int LS, int LO>
cudaError_t launch_conv_fwd(const ConvFwdArgs& a, int num_sms, cudaStream_t stream);
template <int LI, int LS, int LO>
cudaError_t launch_conv_paths(const ConvFwdArgs& a, int num_sms, cudaStream_t stream, int only_l3 = -1);
template <int LI, int LS, int LO>
void conv_path_order(int* order, int* count_l3);
template <int LI, int LS, int LO>
cudaError_t launch_conv_fwd_shared(const ConvFwdArgs& a, int num_sms, cudaStream_t stream);
template <int LI, int LS, int LO>
cudaError_t launch_conv_bwd_shared(const ConvBwdArgs& a, int num_sms, cudaStream_t stream);
template <int LI, int LS, int LO>
cudaError_t launch_conv_bwd_paths(const ConvBwdArgs& a, int num_sms, cudaStream_t stream);
template <int LI, int LS, int LO>
cudaError_t launch_conv_bwd(const ConvBwdArgs& a, int num_sms, cudaStream_t stream);
// The double backward's fused passes (conv_dd.cu) and the number of partial
// slices of each of the fused pass's two harmonic-gradient sets.
template <int LI, int LS, int LO>
cudaError_t launch_conv_dd_fwd(const ConvFwdArgs& a, int num_sms, cudaStream_t stream);
template <int LI, int LS, int LO>
cudaError_t launch_conv_dd_bwd(const ConvBwdArgs& a, int num_sms, cudaStream_t stream);
template <int LI, int LS, int LO>
int conv_dd_slices(int mult);
template <int LI, int LS, int LO>
int conv_bwd_slices(int mult);
template <int LI, int LS, int LO>
cudaError_t launch_tp_fwd(const TPArgs& a, int num_sms, cudaStream_t stream);
template <int LI, int LS, int LO>
cudaError_t launch_tp_bwd(const TPArgs& a, int num_sms, cudaStream_t stream);

cudaError_t launch_graph_build(const float* pos, int n, float box_len, float rc, const int* graph_ptr,
                               int n_graphs, int* row_ptr, int* col, float* edge_vec, int* csc_ptr,
                               int* csc_edge, int* csc_dst, int max_edges, int* n_edges, int num_sms,
                               cudaStream_t stream);
cudaError_t launch_csr_transpose(int n, int n_edges, const int* row_ptr, const int* col, int* csc_ptr,
                                 int* csc_edge, int* csc_dst, int* ws, int num_sms, cudaStream_t stream);
cudaError_t launch_graph_check(int n, int n_edges, const int* row_ptr, const int* col, const float* edge_vec,
                               int* flags, int num_sms, cudaStream_t stream);
// OR the validation bits of the given arrays (each nullable) into *flags.
cudaError_t launch_graph_validate(int n, int n_edges, const int* row_ptr, const int* col, const float* edge_vec,
                                  const int* csc_ptr, const int* csc_edge, const int* csc_dst, int* flags,
                                  int num_sms, cudaStream_t stream);
cudaError_t launch_radial_fwd(int n_edges, int N, const float* ev, float rc, const float* W1, const float* W2,
                              float* w, int num_sms, cudaStream_t stream);
cudaError_t launch_radial_bwd(int n_edges, int N, const float* ev, float rc, const float* W1, const float* W2,
                              const float* gw, float* gev, int num_sms, cudaStream_t stream);
cudaError_t launch_forces(int n, const int* row_ptr, const int* csc_ptr, const int* csc_edge, const float* g,
                          float* F, int num_sms, cudaStream_t stream);
cudaError_t launch_sh(int lmax_sh, int n_edges, const float* ev, float* Y, float* dY, int num_sms,
                      cudaStream_t stream);
// Fully connected convolution, second stage: pack the per-path mixing
// matrices by l3 and multiply (tensor cores, fp32-accurate).
cudaError_t launch_uvw_pack(int n_paths, int mult, int mult_out, int lmax_out, const int* order_dev,
                            const int* count_l3, const float* mix, float* packed, cudaStream_t stream);
size_t uvw_gemm_workspace(int n_nodes, int lmax_out, const int* count_l3, int mult, int mult_out);
cudaError_t launch_uvw_gemm(int n_nodes, int lmax_out, const int* count_l3, int mult, int mult_out,
                            const float* t, const float* packed, float* out, void* ws, size_t ws_bytes,
                            cudaStream_t stream);
// The same GEMMs with each l3 block's producer work first on the block's
// lane: before(l3, lane stream) launches what the block's GEMM reads (its
// per-path messages and packed mixing matrices), so the blocks overlap.
cudaError_t launch_uvw_gemm_after(int n_nodes, int lmax_out, const int* count_l3, int mult, int mult_out,
                                  const float* t, const float* packed, float* out, void* ws, size_t ws_bytes,
                                  cudaStream_t stream, const std::function<cudaError_t(int, cudaStream_t)>& before);
// Packing of one l3 block's mixing matrices (l3 < 0: every block).
cudaError_t launch_uvw_pack_l3(int n_paths, int mult, int mult_out, int lmax_out, const int* order,
                               const int* count_l3, const float* mix, float* packed, int l3, cudaStream_t stream);
cudaError_t launch_uvw_pack_t(int n_paths, int mult, int mult_out, int lmax_out, const int* order,
                              const int* count_l3, const float* mix, float* packed_t, cudaStream_t stream);
size_t uvw_bwd_gemm_workspace(int n_nodes, int lmax_out, const int* count_l3, int mult, int mult_out);
cudaError_t launch_uvw_gt(int n_nodes, int lmax_out, const int* count_l3, int mult, int mult_out, const float* g,
                          const float* packed_t, float* gt, void* ws, size_t ws_bytes, cudaStream_t stream);
cudaError_t launch_uvw_grad_mix(int n_nodes, int n_paths, int lmax_out, const int* order, const int* count_l3,
                                int mult, int mult_out, const float* t, const float* g, float* part,
                                float* grad_mix, void* ws, size_t ws_bytes, cudaStream_t stream);
// dst[k] = src[idx[k]] (add = false) or dst[idx[k]] += src[k] (add = true)
// for n rows of rf floats; idx unique within one call.
cudaError_t launch_rows(bool add, int n, int rf, const int* idx, const float* src, float* dst, int num_sms,
                        cudaStream_t stream);
cudaError_t launch_sh_dir(int lmax_sh, int n_edges, const float* ev, const float* q, float* u, int num_sms,
                          cudaStream_t stream);

}  // namespace cgtp
