// Per-path variants of the convolution kernels for one irreps shape, the
// channelwise stages of the fully connected convolution:
//  - the forward with one block of output rows per path (the messages t
//    that the tensor-core mixing consumes);
//  - the backward with one output gradient per path (the gradients the
//    mixing's transpose produces).
// Both are instantiations of the kernel templates of conv_fwd_kernel.cuh and
// conv_bwd_kernel.cuh.
#include "common.cuh"

namespace cgtp {
CGTP_DEFINE_CONSTANT_TABLES()
}  // namespace cgtp

#include "conv_common.cuh"
#include "vec2.cuh"
#include "sh.cuh"
#include "launch.h"
#include "conv_fwd_kernel.cuh"
#include "conv_bwd_kernel.cuh"

namespace cgtp {
namespace {

// Per-path rows: chunks of same-l3 paths that keep one block of 2 l3 + 1
// output rows per path, at most kPathRowsMax rows per chunk (the
// accumulators stay in registers).
#ifndef CGTP_PATH_ROWS
#define CGTP_PATH_ROWS 16
#endif
constexpr int kPathRowsMax = CGTP_PATH_ROWS;
template <class PS>
using PathPlan = Plan<PS, kByL3, kFwdVec, false, CGTP_FWD_BUDGET, kPathRowsMax>;

template <class PS, class PL, int CH>
struct PathRowsGrp : ChunkGrp<PS, PL, CH, kByL3> {
  using Base = ChunkGrp<PS, PL, CH, kByL3>;
  static constexpr bool PERPATH = true;
  static constexpr int NOWN = Base::NP * (2 * Base::KEY + 1);
  static constexpr int key_first() {  // first place of this l3 in the plan's order
    for (int c = 0; c < PL::P.n; ++c)
      if (PL::P.key[c] == Base::KEY) return PL::P.first[c];
    return 0;
  }
  static constexpr int key_count() {
    int n = 0;
    for (int c = 0; c < PL::P.n; ++c)
      if (PL::P.key[c] == Base::KEY) n += PL::P.count[c];
    return n;
  }
  static constexpr int NPK = key_count();                    // paths with this l3
  static constexpr int PL0 = PL::P.first[CH] - key_first();  // rank of the chunk's first path
};

}  // namespace

// Paths in the order of the per-path rows (by l3, then l2, then
// lexicographic) and the number of paths of each l3.
template <int LI, int LS, int LO>
void conv_path_order(int* order, int* count_l3) {
  using PL = PathPlan<PathSet<LI, LS, LO>>;
  for (int l = 0; l <= LO; ++l) count_l3[l] = 0;
  int k = 0;
  for (int c = 0; c < PL::P.n; ++c)
    for (int q = 0; q < PL::P.count[c]; ++q) {
      order[k++] = PL::P.order[PL::P.first[c] + q];
      ++count_l3[PL::P.key[c]];
    }
}

// Per-path messages t: a.out is t, whose block for l3 holds
// [n_nodes][2 l3 + 1][paths of l3][mult] and follows the blocks of smaller l3.
// only_l3 >= 0: the chunks of that l3 block alone (the fully connected
// forward runs each block's chunks on its own lane, ahead of its GEMM).
template <int LI, int LS, int LO>
cudaError_t launch_conv_paths(const ConvFwdArgs& a, int num_sms, cudaStream_t stream, int only_l3) {
  using PS = PathSet<LI, LS, LO>;
  using PL = PathPlan<PS>;
  cudaError_t err = cudaSuccess;
  bool first = true;
  static_for_host<0, PL::N>([&](auto Cc) {
    constexpr int CH = decltype(Cc)::value;
    using GR = PathRowsGrp<PS, PL, CH>;
    if (only_l3 >= 0 && GR::KEY != only_l3) return;
    size_t off = 0;  // floats before the l3 = KEY block
    for (int c = 0; c < PL::P.n; ++c)
      if (PL::P.key[c] < GR::KEY) off += (size_t)PL::P.count[c] * (2 * PL::P.key[c] + 1);
    ConvFwdArgs b = a;
    b.out = a.out + off * (size_t)a.n_nodes * a.mult;
    b.accumulate = 0;
    // chunks write disjoint rows: all but the first launched may overlap the one before
    if (err == cudaSuccess) err = launch_fwd_group<PS, GR, false>(b, num_sms, !first, stream);
    first = false;
  });
  return err;
}

template <int LI, int LS, int LO>
cudaError_t launch_conv_bwd_paths(const ConvBwdArgs& a, int num_sms, cudaStream_t stream) {
  return launch_bwd_all<PathSet<LI, LS, LO>, kVarPerPath, true>(a, num_sms, stream);
}

// One translation unit per shape (the build passes CGTP_CFG_LI/LS/LO).
template cudaError_t launch_conv_paths<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(const ConvFwdArgs&, int,
                                                                           cudaStream_t, int);
template void conv_path_order<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(int*, int*);
template cudaError_t launch_conv_bwd_paths<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(const ConvBwdArgs&, int,
                                                                                cudaStream_t);

}  // namespace cgtp
