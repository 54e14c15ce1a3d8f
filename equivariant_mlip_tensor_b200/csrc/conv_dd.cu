// The double backward's fused passes for one irreps shape: the forward that
// gives d grad_out and the source-centric pass that gives d x, d W and the
// edge-vector term, with W and gg_W read once per pass.  Instantiations of
// the kernel templates of conv_fwd_kernel.cuh and conv_bwd_kernel.cuh
// (variants DD and kVarDD).
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
cudaError_t launch_conv_dd_fwd(const ConvFwdArgs& a, int num_sms, cudaStream_t stream) {
  return launch_fwd_dd<PathSet<LI, LS, LO>>(a, num_sms, stream);
}

template <int LI, int LS, int LO>
cudaError_t launch_conv_dd_bwd(const ConvBwdArgs& a, int num_sms, cudaStream_t stream) {
  return launch_bwd_dd<PathSet<LI, LS, LO>>(a, num_sms, stream);
}

template <int LI, int LS, int LO>
int conv_dd_slices(int mult) {
  return bwd_slices<PathSet<LI, LS, LO>, kVarDD>(mult);
}

// One translation unit per shape (the build passes CGTP_CFG_LI/LS/LO).
template cudaError_t launch_conv_dd_fwd<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(const ConvFwdArgs&, int,
                                                                            cudaStream_t);
template cudaError_t launch_conv_dd_bwd<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(const ConvBwdArgs&, int,
                                                                            cudaStream_t);
template int conv_dd_slices<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(int);

}  // namespace cgtp
