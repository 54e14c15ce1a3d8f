// Irreps shapes (lmax_in, lmax_sh, lmax_out) whose kernels are compiled in.
//
// CGTP_CONFIGS: the channelwise convolution (forward, backward, double
// backward) and the edge-free pair product with its CP surrogate.  Policy:
// every shape with lmax_in, lmax_out <= 3 and lmax_sh <= 4 that is
//   - an interaction layer (lmax_in == lmax_out), or
//   - an embedding layer (lmax_in == 0: scalar inputs to any output), or
//   - a read-out layer (lmax_out == 0: any input to scalar outputs);
// 50 shapes.  CGTP_VARIANT_CONFIGS: the weight-structure variants (weights
// shared by every path, the fully connected convolution), built for the
// shapes of the standard workloads only.  Every kernel family is
// instantiated for each entry of its list; the C ABI reports any other
// shape as unsupported (cgtp_supported).  tests/test_abi_cpu.py checks both
// lists against the policy.
#pragma once

#define CGTP_CONFIGS(X)                                                            \
  X(0, 0, 0) X(0, 1, 0) X(0, 2, 0) X(0, 3, 0) X(0, 4, 0)                          \
  X(0, 0, 1) X(0, 1, 1) X(0, 2, 1) X(0, 3, 1) X(0, 4, 1)                          \
  X(0, 0, 2) X(0, 1, 2) X(0, 2, 2) X(0, 3, 2) X(0, 4, 2)                          \
  X(0, 0, 3) X(0, 1, 3) X(0, 2, 3) X(0, 3, 3) X(0, 4, 3)                          \
  X(1, 0, 0) X(1, 1, 0) X(1, 2, 0) X(1, 3, 0) X(1, 4, 0)                          \
  X(2, 0, 0) X(2, 1, 0) X(2, 2, 0) X(2, 3, 0) X(2, 4, 0)                          \
  X(3, 0, 0) X(3, 1, 0) X(3, 2, 0) X(3, 3, 0) X(3, 4, 0)                          \
  X(1, 0, 1) X(1, 1, 1) X(1, 2, 1) X(1, 3, 1) X(1, 4, 1)                          \
  X(2, 0, 2) X(2, 1, 2) X(2, 2, 2) X(2, 3, 2) X(2, 4, 2)                          \
  X(3, 0, 3) X(3, 1, 3) X(3, 2, 3) X(3, 3, 3) X(3, 4, 3)

#define CGTP_VARIANT_CONFIGS(X) \
  X(0, 0, 0) X(1, 1, 1) X(1, 2, 1) X(2, 2, 2) X(2, 4, 2) X(3, 3, 3)
