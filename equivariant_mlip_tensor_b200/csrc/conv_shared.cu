// Convolution with one weight row per edge shared by every path (path
// stride 0: W_e[p][u] = w_e[u]), forward and backward, for one irreps shape:
//   out[i][l3,m3][u] = sum_{e in row i} w_e[u] sum_p sum_{m1,m2} C^p x[j][l1,m1][u] Y_e[l2,m2]
//   grad_w[e][u]     = sum_p (the per-path weight gradient of the channelwise convolution)
// ("Tensor Decomposition Networks ...", reply to reviewer oXft: weights shared
// across paths).  Instantiations of the kernel templates of
// conv_fwd_kernel.cuh and conv_bwd_kernel.cuh with one staged weight row per
// edge; the backward's chunks run in plain stream order because each adds
// onto the gradient rows the previous chunks wrote.
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

template <int LI, int LS, int LO>
cudaError_t launch_conv_fwd_shared(const ConvFwdArgs& a, int num_sms, cudaStream_t stream) {
  return launch_fwd_all<PathSet<LI, LS, LO>, true>(a, num_sms, stream);
}

template <int LI, int LS, int LO>
cudaError_t launch_conv_bwd_shared(const ConvBwdArgs& a, int num_sms, cudaStream_t stream) {
  if (a.sh != nullptr || a.accumulate) return cudaErrorInvalidValue;
  return launch_bwd_all<PathSet<LI, LS, LO>, kVarWShared, false>(a, num_sms, stream);
}

// One translation unit per shape (the build passes CGTP_CFG_LI/LS/LO).
template cudaError_t launch_conv_fwd_shared<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(const ConvFwdArgs&, int,
                                                                                cudaStream_t);
template cudaError_t launch_conv_bwd_shared<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(const ConvBwdArgs&, int,
                                                                                cudaStream_t);

}  // namespace cgtp
