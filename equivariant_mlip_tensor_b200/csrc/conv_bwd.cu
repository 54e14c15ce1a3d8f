// Convolution backward (per-path weights): the instantiation of the backward
// kernel template for one irreps shape, with the l1 blocks on forked lanes.
// The double backward's first-order passes (caller harmonics, accumulate)
// select the kVarExt kernel at run time.
#include "common.cuh"

namespace cgtp {
CGTP_DEFINE_CONSTANT_TABLES()
}  // namespace cgtp

#include "conv_common.cuh"
#include "vec2.cuh"
#include "sh.cuh"
#include "launch.h"
#include "conv_bwd_kernel.cuh"

namespace cgtp {

#ifndef CGTP_BWD_LANES
#define CGTP_BWD_LANES 1
#endif

template <int LI, int LS, int LO>
int conv_bwd_slices(int mult) {
  return bwd_slices<PathSet<LI, LS, LO>>(mult);
}

template <int LI, int LS, int LO>
cudaError_t launch_conv_bwd(const ConvBwdArgs& a, int num_sms, cudaStream_t stream) {
  return launch_bwd_all<PathSet<LI, LS, LO>, 0, CGTP_BWD_LANES != 0>(a, num_sms, stream);
}

// One translation unit per shape (the build passes CGTP_CFG_LI/LS/LO).
template cudaError_t launch_conv_bwd<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(const ConvBwdArgs&, int,
                                                                         cudaStream_t);
template int conv_bwd_slices<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(int);

}  // namespace cgtp
