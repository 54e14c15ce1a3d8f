// Fully connected ("uvw") convolution, second stage: per l3 block,
//   out[i][l3, m3][v] = sum_{p: l3(p) = l3} sum_u t[i][p][m3][u] mix[p][u][v]
// is one dense GEMM with the block's paths concatenated along K
// (K = paths x mult), batched over m3 ("Tensor Decomposition Networks ...",
// reply to reviewer cmnz: the fully connected CG tensor product).  The GEMM
// runs on the 5th-generation tensor cores through CUTLASS's sm100 collective
// (TMA-staged operands, tcgen05 MMA into tensor memory) in its fp32-accurate
// mode: each fp32 operand is split into three bf16 terms and, of the nine
// products, the six above fp32 rounding are accumulated in fp32, which keeps
// the result within fp32 rounding of the exact product.  Cluster shape 1x1x1: every CTA loads its own
// operand tiles from this GPU's memory.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "launch.h"

#if !defined(CGTP_NO_CUTLASS)
#include "cutlass/cutlass.h"
#include "cute/tensor.hpp"
#include "cutlass/epilogue/collective/collective_builder.hpp"
#include "cutlass/gemm/collective/collective_builder.hpp"
#include "cutlass/gemm/device/gemm_universal_adapter.h"
#include "cutlass/gemm/dispatch_policy.hpp"
#include "cutlass/gemm/kernel/gemm_universal.hpp"
#include "cutlass/util/packed_stride.hpp"
#endif

namespace cgtp {

namespace {

struct PathOrder {
  int order[kMaxPaths];  // path of each rank, ranks grouped by l3
};

// packed block of l3: [2 l3 + 1 copies][paths of l3 x mult][mult_out]
__global__ void uvw_pack_kernel(PathOrder po, int mult, int mult_out, int rank0, int npk, int n3,
                                const float* __restrict__ mix, float* __restrict__ packed) {
  const long long per_copy = (long long)npk * mult * mult_out;
  const long long total = per_copy * n3;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long r = i % per_copy;
    const int v = int(r % mult_out);
    const long long ku = r / mult_out;
    const int uu = int(ku % mult), rank = int(ku / mult);
    packed[i] = mix[((long long)po.order[rank0 + rank] * mult + uu) * mult_out + v];
  }
}

// packed transposed block of l3: [2 l3 + 1 copies][mult_out][paths of l3 x mult]
__global__ void uvw_pack_t_kernel(PathOrder po, int mult, int mult_out, int rank0, int npk, int n3,
                                  const float* __restrict__ mix, float* __restrict__ packed) {
  const long long K = (long long)npk * mult;
  const long long per_copy = K * mult_out;
  const long long total = per_copy * n3;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long r = i % per_copy;
    const long long ku = r % K;
    const int v = int(r / K);
    const int uu = int(ku % mult), rank = int(ku / mult);
    packed[i] = mix[((long long)po.order[rank0 + rank] * mult + uu) * mult_out + v];
  }
}

// grad_mix[p][u][v] = sum_m3 part[m3][rank(p) * mult + u][v] for the paths of one l3 block
__global__ void uvw_unpack_kernel(PathOrder po, int mult, int mult_out, int rank0, int npk, int n3,
                                  const float* __restrict__ part, float* __restrict__ grad_mix) {
  const long long K = (long long)npk * mult;
  const long long total = K * mult_out;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int m3 = 0; m3 < n3; ++m3) s += part[m3 * total + i];
    const int v = int(i % mult_out);
    const long long ku = i / mult_out;
    const int uu = int(ku % mult), rank = int(ku / mult);
    grad_mix[((long long)po.order[rank0 + rank] * mult + uu) * mult_out + v] = s;
  }
}

// The GEMMs of the l3 blocks are independent (disjoint outputs): they run
// concurrently, block l3 on lane l3 % kLanes of a fork from the caller's
// stream (lane 0 is the caller's stream itself) and join back before the
// call returns, so the caller sees ordinary stream order.  The side streams
// and events are the library's per-device pool (lanes.cu).
constexpr int kLanes = 3;
using Lanes = SideLanes;
static cudaError_t lanes_for_device(Lanes** out) { return side_lanes(kLanesUvw, out); }
static cudaError_t lanes_fork(Lanes* L, cudaStream_t s) { return lanes_fork(L, kLanes - 1, s); }
static cudaError_t lanes_join(Lanes* L, cudaStream_t s) { return lanes_join(L, kLanes - 1, s); }
static cudaStream_t lane(Lanes* L, cudaStream_t s, int l3) { return l3 % kLanes == 0 ? s : L->side[l3 % kLanes - 1]; }
// Host threads that enqueue on the shared lanes take turns (the fork and join
// events are shared too).
static std::mutex& lanes_use_mutex() { return side_lanes_mutex(kLanesUvw); }

#if !defined(CGTP_NO_CUTLASS)
using namespace cute;
#ifndef CGTP_UVW_TILE_N
#define CGTP_UVW_TILE_N 128  // output-channel tile of the mixing GEMMs
#endif
#ifndef CGTP_UVW_TILE_N_MIX
#define CGTP_UVW_TILE_N_MIX 64  // mixing-gradient GEMM: few, long tiles, so narrower ones
#endif
#ifndef CGTP_UVW_TILE_M
#define CGTP_UVW_TILE_M 128  // node-row tile of the mixing GEMMs
#endif
using TileShape = Shape<Int<CGTP_UVW_TILE_M>, Int<CGTP_UVW_TILE_N>, _32>;
using TileShapeT = Shape<_128, Int<CGTP_UVW_TILE_N_MIX>, _32>;
using ClusterShape = Shape<_1, _1, _1>;
constexpr int kAlign = 4;  // floats: 16-byte rows and strides
using Layout = cutlass::layout::RowMajor;
using Epilogue = typename cutlass::epilogue::collective::CollectiveBuilder<
    cutlass::arch::Sm100, cutlass::arch::OpClassTensorOp, TileShape, ClusterShape,
    cutlass::epilogue::collective::EpilogueTileAuto, float, float, float, Layout, kAlign, float, Layout, kAlign,
    cutlass::epilogue::collective::EpilogueScheduleAuto>::CollectiveOp;
// Product bands of the fp32-accurate mode: each operand is split into three
// bf16 terms x = x0 + x1 + x2 (|x1| <= 2^-9 |x|, |x2| <= 2^-18 |x|), and band
// k holds the products x_i y_j with i + j = k.  Bands 0..2 (six products)
// leave out terms below 2^-26 |x y|, under fp32 rounding; the library's
// builder computes all five (nine products).  Three bands: molecules forward
// 0.517 -> 0.510 ms.
#ifndef CGTP_UVW_BANDS
#define CGTP_UVW_BANDS 3
#endif
template <int NB, class CM>
struct WithBands {
  using type = CM;
};
template <int NB, int L2T, int T2M, int SP, int AP, int NB0, int SF, int PI, class Cl, class Cp, class Ar,
          class... Rest>
struct WithBands<NB, cutlass::gemm::collective::CollectiveMma<
                         cutlass::gemm::MainloopSm100TmaUmmaWarpSpecializedFastF32<L2T, T2M, SP, AP, NB0, SF, PI, Cl,
                                                                                   Cp, Ar>,
                         Rest...>> {
  using type = cutlass::gemm::collective::CollectiveMma<
      cutlass::gemm::MainloopSm100TmaUmmaWarpSpecializedFastF32<L2T, T2M, SP, AP, NB, SF, PI, Cl, Cp, Ar>, Rest...>;
};
using Mainloop = typename WithBands<
    CGTP_UVW_BANDS,
    typename cutlass::gemm::collective::CollectiveBuilder<
        cutlass::arch::Sm100, cutlass::arch::OpClassTensorOp, float, Layout, kAlign, float, Layout, kAlign, float,
        TileShape, ClusterShape,
        cutlass::gemm::collective::StageCountAutoCarveout<static_cast<int>(sizeof(typename Epilogue::SharedStorage))>,
        cutlass::gemm::KernelTmaWarpSpecialized1SmFastFP32Sm100>::CollectiveOp>::type;
static_assert(CGTP_UVW_BANDS == 5 || !std::is_same_v<Mainloop,
                                                      typename cutlass::gemm::collective::CollectiveBuilder<
                                                          cutlass::arch::Sm100, cutlass::arch::OpClassTensorOp, float,
                                                          Layout, kAlign, float, Layout, kAlign, float, TileShape,
                                                          ClusterShape,
                                                          cutlass::gemm::collective::StageCountAutoCarveout<
                                                              static_cast<int>(sizeof(typename Epilogue::SharedStorage))>,
                                                          cutlass::gemm::KernelTmaWarpSpecialized1SmFastFP32Sm100>::CollectiveOp>,
              "the band count did not reach the mainloop");
using Kernel = cutlass::gemm::kernel::GemmUniversal<Shape<int, int, int, int>, Mainloop, Epilogue>;
using Gemm = cutlass::gemm::device::GemmUniversalAdapter<Kernel>;

// Arguments of the GEMM of one l3 block: A = t block [n_nodes][n3][K] read
// as n3 batches of [n_nodes][K] (row stride n3 K, batch stride K); B = the
// packed copies [n3][K][mult_out]; D = out rows (l3, m3) of every node (row
// stride NO mult_out, batch stride mult_out).
// D = A^T B with A stored K-major (column-major A): the mixing-matrix gradient.
using LayoutCol = cutlass::layout::ColumnMajor;
using EpilogueT = typename cutlass::epilogue::collective::CollectiveBuilder<
    cutlass::arch::Sm100, cutlass::arch::OpClassTensorOp, TileShapeT, ClusterShape,
    cutlass::epilogue::collective::EpilogueTileAuto, float, float, float, Layout, kAlign, float, Layout, kAlign,
    cutlass::epilogue::collective::EpilogueScheduleAuto>::CollectiveOp;
using MainloopT = typename WithBands<
    CGTP_UVW_BANDS,
    typename cutlass::gemm::collective::CollectiveBuilder<
        cutlass::arch::Sm100, cutlass::arch::OpClassTensorOp, float, LayoutCol, kAlign, float, Layout, kAlign, float,
        TileShapeT, ClusterShape,
        cutlass::gemm::collective::StageCountAutoCarveout<static_cast<int>(sizeof(typename EpilogueT::SharedStorage))>,
        cutlass::gemm::KernelTmaWarpSpecialized1SmFastFP32Sm100>::CollectiveOp>::type;
using KernelT = cutlass::gemm::kernel::GemmUniversal<Shape<int, int, int, int>, MainloopT, EpilogueT>;
using GemmT = cutlass::gemm::device::GemmUniversalAdapter<KernelT>;

// gt block l3 = grad_out rows (l3, m3) x packed^T: A = grad_out [n_nodes][v] per
// m3 batch (row stride NO v, batch stride v), B = [n3][v][K], D = gt block
// [n_nodes][n3][K] (row stride n3 K, batch stride K).
Gemm::Arguments block_args_gt(int n_nodes, int l3, int lmax_out, int K, int mult_out, const float* g,
                              const float* packed_t, float* gt) {
  const int n3 = 2 * l3 + 1, no = (lmax_out + 1) * (lmax_out + 1);
  using SA = typename Kernel::StrideA;
  using SB = typename Kernel::StrideB;
  using SC = typename Kernel::StrideC;
  using SD = typename Kernel::StrideD;
  SA sa = cutlass::make_cute_packed_stride(SA{}, make_shape(n_nodes, mult_out, n3));
  get<0>(sa) = (int64_t)no * mult_out;
  get<2>(sa) = mult_out;
  SB sb = cutlass::make_cute_packed_stride(SB{}, make_shape(K, mult_out, n3));
  SD sd = cutlass::make_cute_packed_stride(SD{}, make_shape(n_nodes, K, n3));
  get<0>(sd) = (int64_t)n3 * K;
  get<2>(sd) = K;
  SC sc = sd;
  const float* A = g == nullptr ? nullptr : g + (size_t)l3 * l3 * mult_out;
  return Gemm::Arguments{cutlass::gemm::GemmUniversalMode::kGemm,
                         {n_nodes, K, mult_out, n3},
                         {A, sa, packed_t, sb},
                         {{1.f, 0.f}, gt, sc, gt, sd}};
}

// part[m3] = t block (m3)^T x grad_out rows (l3, m3): A = t viewed K-major
// (column-major [K][n_nodes], column stride n3 K, batch stride K), B =
// grad_out [n_nodes][v] (row stride NO v, batch stride v), D = [n3][K][v].
GemmT::Arguments block_args_mix(int n_nodes, int l3, int lmax_out, int K, int mult_out, const float* t,
                                const float* g, float* part) {
  const int n3 = 2 * l3 + 1, no = (lmax_out + 1) * (lmax_out + 1);
  using SA = typename KernelT::StrideA;
  using SB = typename KernelT::StrideB;
  using SC = typename KernelT::StrideC;
  using SD = typename KernelT::StrideD;
  SA sa = cutlass::make_cute_packed_stride(SA{}, make_shape(K, n_nodes, n3));
  get<1>(sa) = (int64_t)n3 * K;
  get<2>(sa) = K;
  SB sb = cutlass::make_cute_packed_stride(SB{}, make_shape(mult_out, n_nodes, n3));
  get<1>(sb) = (int64_t)no * mult_out;
  get<2>(sb) = mult_out;
  SD sd = cutlass::make_cute_packed_stride(SD{}, make_shape(K, mult_out, n3));
  SC sc = sd;
  const float* B = g == nullptr ? nullptr : g + (size_t)l3 * l3 * mult_out;
  return GemmT::Arguments{cutlass::gemm::GemmUniversalMode::kGemm,
                          {K, mult_out, n_nodes, n3},
                          {t, sa, B, sb},
                          {{1.f, 0.f}, part, sc, part, sd}};
}

Gemm::Arguments block_args(int n_nodes, int l3, int lmax_out, int K, int mult_out, const float* t,
                           const float* packed, float* out) {
  const int n3 = 2 * l3 + 1, no = (lmax_out + 1) * (lmax_out + 1);
  using SA = typename Kernel::StrideA;
  using SB = typename Kernel::StrideB;
  using SC = typename Kernel::StrideC;
  using SD = typename Kernel::StrideD;
  SA sa = cutlass::make_cute_packed_stride(SA{}, make_shape(n_nodes, K, n3));
  get<0>(sa) = (int64_t)n3 * K;
  get<2>(sa) = K;
  SB sb = cutlass::make_cute_packed_stride(SB{}, make_shape(mult_out, K, n3));
  SD sd = cutlass::make_cute_packed_stride(SD{}, make_shape(n_nodes, mult_out, n3));
  get<0>(sd) = (int64_t)no * mult_out;
  get<2>(sd) = mult_out;
  SC sc = sd;
  float* D = out + (size_t)l3 * l3 * mult_out;
  return Gemm::Arguments{cutlass::gemm::GemmUniversalMode::kGemm,
                         {n_nodes, mult_out, K, n3},
                         {t, sa, packed, sb},
                         {{1.f, 0.f}, D, sc, D, sd}};
}
#endif

}  // namespace

cudaError_t launch_uvw_pack_l3(int n_paths, int mult, int mult_out, int lmax_out, const int* order,
                               const int* count_l3, const float* mix, float* packed, int only_l3,
                               cudaStream_t stream) {
  PathOrder po{};
  for (int k = 0; k < n_paths && k < kMaxPaths; ++k) po.order[k] = order[k];
  int rank0 = 0;
  size_t off = 0;
  for (int l3 = 0; l3 <= lmax_out; ++l3) {
    const int npk = count_l3[l3], n3 = 2 * l3 + 1;
    if (npk > 0 && (only_l3 < 0 || l3 == only_l3)) {
      uvw_pack_kernel<<<256, 256, 0, stream>>>(po, mult, mult_out, rank0, npk, n3, mix, packed + off);
      const cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    off += (size_t)n3 * npk * mult * mult_out;
    rank0 += npk;
  }
  return cudaSuccess;
}

cudaError_t launch_uvw_pack(int n_paths, int mult, int mult_out, int lmax_out, const int* order, const int* count_l3,
                            const float* mix, float* packed, cudaStream_t stream) {
  return launch_uvw_pack_l3(n_paths, mult, mult_out, lmax_out, order, count_l3, mix, packed, -1, stream);
}

size_t uvw_gemm_workspace(int n_nodes, int lmax_out, const int* count_l3, int mult, int mult_out) {
#if defined(CGTP_NO_CUTLASS)
  return 0;
#else
  size_t w = 0;
  for (int l3 = 0; l3 <= lmax_out; ++l3) {
    if (count_l3[l3] == 0) continue;
    const size_t b = Gemm::get_workspace_size(
        block_args(n_nodes, l3, lmax_out, count_l3[l3] * mult, mult_out, nullptr, nullptr, nullptr));
    w = b > w ? b : w;
  }
  return kLanes * ((w + 255) & ~(size_t)255);  // one slice per lane
#endif
}

cudaError_t launch_uvw_gemm_after(int n_nodes, int lmax_out, const int* count_l3, int mult, int mult_out,
                                  const float* t, const float* packed, float* out, void* ws, size_t ws_bytes,
                                  cudaStream_t stream,
                                  const std::function<cudaError_t(int, cudaStream_t)>& before) {
#if defined(CGTP_NO_CUTLASS)
  return cudaErrorNotSupported;
#else
  std::lock_guard<std::mutex> turn(lanes_use_mutex());
  Lanes* Ls = nullptr;
  cudaError_t e = lanes_for_device(&Ls);
  if (e == cudaSuccess) e = lanes_fork(Ls, stream);
  if (e != cudaSuccess) return e;
  const size_t slice = (ws_bytes / kLanes) & ~(size_t)255;
  size_t t_off = 0, p_off = 0;
  for (int l3 = 0; l3 <= lmax_out && e == cudaSuccess; ++l3) {
    const int npk = count_l3[l3], n3 = 2 * l3 + 1, K = npk * mult;
    cudaStream_t st = lane(Ls, stream, l3);
    if (before) e = before(l3, st);
    if (npk > 0 && e == cudaSuccess) {
      void* w = (char*)ws + (size_t)(l3 % kLanes) * slice;
      Gemm g;
      auto args = block_args(n_nodes, l3, lmax_out, K, mult_out, t + t_off, packed + p_off, out);
      if (g.can_implement(args) != cutlass::Status::kSuccess) e = cudaErrorNotSupported;
      else if (Gemm::get_workspace_size(args) > slice) e = cudaErrorInvalidValue;
      else if (g.initialize(args, w, st) != cutlass::Status::kSuccess) e = cudaErrorLaunchFailure;
      else if (g.run(st) != cutlass::Status::kSuccess) e = cudaErrorLaunchFailure;
    }
    t_off += (size_t)n_nodes * n3 * K;
    p_off += (size_t)n3 * K * mult_out;
  }
  const cudaError_t ej = lanes_join(Ls, stream);
  if (e != cudaSuccess) return e;
  return ej != cudaSuccess ? ej : cudaGetLastError();
#endif
}

cudaError_t launch_uvw_gemm(int n_nodes, int lmax_out, const int* count_l3, int mult, int mult_out, const float* t,
                            const float* packed, float* out, void* ws, size_t ws_bytes, cudaStream_t stream) {
  return launch_uvw_gemm_after(n_nodes, lmax_out, count_l3, mult, mult_out, t, packed, out, ws, ws_bytes, stream,
                               nullptr);
}

cudaError_t launch_uvw_pack_t(int n_paths, int mult, int mult_out, int lmax_out, const int* order,
                              const int* count_l3, const float* mix, float* packed_t, cudaStream_t stream) {
  PathOrder po{};
  for (int k = 0; k < n_paths && k < kMaxPaths; ++k) po.order[k] = order[k];
  int rank0 = 0;
  size_t off = 0;
  for (int l3 = 0; l3 <= lmax_out; ++l3) {
    const int npk = count_l3[l3], n3 = 2 * l3 + 1;
    if (npk > 0) {
      uvw_pack_t_kernel<<<256, 256, 0, stream>>>(po, mult, mult_out, rank0, npk, n3, mix, packed_t + off);
      const cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    off += (size_t)n3 * npk * mult * mult_out;
    rank0 += npk;
  }
  return cudaSuccess;
}

size_t uvw_bwd_gemm_workspace(int n_nodes, int lmax_out, const int* count_l3, int mult, int mult_out) {
#if defined(CGTP_NO_CUTLASS)
  return 0;
#else
  size_t w = 0;
  for (int l3 = 0; l3 <= lmax_out; ++l3) {
    if (count_l3[l3] == 0) continue;
    const int K = count_l3[l3] * mult;
    const size_t a = Gemm::get_workspace_size(block_args_gt(n_nodes, l3, lmax_out, K, mult_out, nullptr, nullptr,
                                                            nullptr));
    const size_t b = GemmT::get_workspace_size(block_args_mix(n_nodes, l3, lmax_out, K, mult_out, nullptr, nullptr,
                                                              nullptr));
    w = a > w ? a : w;
    w = b > w ? b : w;
  }
  return kLanes * ((w + 255) & ~(size_t)255);  // one slice per lane
#endif
}

// gt = per-path output gradients (per l3 block: grad_out rows x packed^T)
cudaError_t launch_uvw_gt(int n_nodes, int lmax_out, const int* count_l3, int mult, int mult_out, const float* g,
                          const float* packed_t, float* gt, void* ws, size_t ws_bytes, cudaStream_t stream) {
#if defined(CGTP_NO_CUTLASS)
  return cudaErrorNotSupported;
#else
  std::lock_guard<std::mutex> turn(lanes_use_mutex());
  Lanes* Ls = nullptr;
  cudaError_t e = lanes_for_device(&Ls);
  if (e == cudaSuccess) e = lanes_fork(Ls, stream);
  if (e != cudaSuccess) return e;
  const size_t slice = (ws_bytes / kLanes) & ~(size_t)255;
  size_t t_off = 0, p_off = 0;
  for (int l3 = 0; l3 <= lmax_out && e == cudaSuccess; ++l3) {
    const int npk = count_l3[l3], n3 = 2 * l3 + 1, K = npk * mult;
    if (npk > 0) {
      cudaStream_t st = lane(Ls, stream, l3);
      void* w = (char*)ws + (size_t)(l3 % kLanes) * slice;
      Gemm gm;
      auto args = block_args_gt(n_nodes, l3, lmax_out, K, mult_out, g, packed_t + p_off, gt + t_off);
      if (gm.can_implement(args) != cutlass::Status::kSuccess) e = cudaErrorNotSupported;
      else if (Gemm::get_workspace_size(args) > slice) e = cudaErrorInvalidValue;
      else if (gm.initialize(args, w, st) != cutlass::Status::kSuccess) e = cudaErrorLaunchFailure;
      else if (gm.run(st) != cutlass::Status::kSuccess) e = cudaErrorLaunchFailure;
    }
    t_off += (size_t)n_nodes * n3 * K;
    p_off += (size_t)n3 * K * mult_out;
  }
  const cudaError_t ej = lanes_join(Ls, stream);
  if (e != cudaSuccess) return e;
  return ej != cudaSuccess ? ej : cudaGetLastError();
#endif
}

// grad_mix from the per-path messages t and grad_out (per l3 block, one
// partial per m3 summed by the unpacking kernel); part: [sum_l3 n3 K v] floats
cudaError_t launch_uvw_grad_mix(int n_nodes, int n_paths, int lmax_out, const int* order, const int* count_l3,
                                int mult, int mult_out, const float* t, const float* g, float* part,
                                float* grad_mix, void* ws, size_t ws_bytes, cudaStream_t stream) {
#if defined(CGTP_NO_CUTLASS)
  return cudaErrorNotSupported;
#else
  PathOrder po{};
  for (int k = 0; k < n_paths && k < kMaxPaths; ++k) po.order[k] = order[k];
  std::lock_guard<std::mutex> turn(lanes_use_mutex());
  Lanes* Ls = nullptr;
  cudaError_t e = lanes_for_device(&Ls);
  if (e == cudaSuccess) e = lanes_fork(Ls, stream);
  if (e != cudaSuccess) return e;
  const size_t slice = (ws_bytes / kLanes) & ~(size_t)255;
  size_t t_off = 0, p_off = 0;
  int rank0 = 0;
  for (int l3 = 0; l3 <= lmax_out && e == cudaSuccess; ++l3) {
    const int npk = count_l3[l3], n3 = 2 * l3 + 1, K = npk * mult;
    if (npk > 0) {
      cudaStream_t st = lane(Ls, stream, l3);
      void* w = (char*)ws + (size_t)(l3 % kLanes) * slice;
      GemmT gm;
      auto args = block_args_mix(n_nodes, l3, lmax_out, K, mult_out, t + t_off, g, part + p_off);
      if (gm.can_implement(args) != cutlass::Status::kSuccess) e = cudaErrorNotSupported;
      else if (GemmT::get_workspace_size(args) > slice) e = cudaErrorInvalidValue;
      else if (gm.initialize(args, w, st) != cutlass::Status::kSuccess) e = cudaErrorLaunchFailure;
      else if (gm.run(st) != cutlass::Status::kSuccess) e = cudaErrorLaunchFailure;
      if (e == cudaSuccess) {
        uvw_unpack_kernel<<<256, 256, 0, st>>>(po, mult, mult_out, rank0, npk, n3, part + p_off, grad_mix);
        e = cudaGetLastError();
      }
    }
    t_off += (size_t)n_nodes * n3 * K;
    p_off += (size_t)n3 * K * mult_out;
    rank0 += npk;
  }
  const cudaError_t ej = lanes_join(Ls, stream);
  if (e != cudaSuccess) return e;
  return ej != cudaSuccess ? ej : cudaGetLastError();
#endif
}

}  // namespace cgtp
