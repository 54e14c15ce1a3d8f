// The harmonic gradient alone (grad_x and grad_W not wanted), for the double
// backward's passes that need grad_Y only: the chunks of the plain backward
// without the T^T g products (kVarGyOnly), then the Jacobian epilogue of
// a.gr_mode.  Partials go to a.grad_sh in the plain backward's layout (the
// same chunks and slices).  An instantiation of the kernel template of
// conv_bwd_kernel.cuh for one irreps shape.
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

template <int LI, int LS, int LO>
cudaError_t launch_conv_bwd_gy(const ConvBwdArgs& a, int num_sms, cudaStream_t stream) {
  return launch_bwd_all<PathSet<LI, LS, LO>, kVarGyOnly, true>(a, num_sms, stream);
}

// One translation unit per shape (the build passes CGTP_CFG_LI/LS/LO).
template cudaError_t launch_conv_bwd_gy<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(const ConvBwdArgs&, int,
                                                                             cudaStream_t);

}  // namespace cgtp
