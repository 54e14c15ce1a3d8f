// Convolution forward (per-path weights, paths summed into l3 blocks): the
// instantiation of the forward kernel template for one irreps shape.
#include "common.cuh"

namespace cgtp {
CGTP_DEFINE_CONSTANT_TABLES()
}  // namespace cgtp

#include "conv_common.cuh"
#include "vec2.cuh"
#include "sh.cuh"
#include "launch.h"
#include "conv_fwd_kernel.cuh"

namespace cgtp {

template <int LI, int LS, int LO>
cudaError_t launch_conv_fwd(const ConvFwdArgs& a, int num_sms, cudaStream_t stream) {
  return launch_fwd_all<PathSet<LI, LS, LO>, false>(a, num_sms, stream);
}

// One translation unit per shape (the build passes CGTP_CFG_LI/LS/LO).
template cudaError_t launch_conv_fwd<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(const ConvFwdArgs&, int,
                                                                         cudaStream_t);

}  // namespace cgtp
