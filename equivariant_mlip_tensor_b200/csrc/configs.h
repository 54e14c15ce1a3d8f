// Irreps shapes (lmax_in, lmax_sh, lmax_out) whose kernels are compiled in.
// Every kernel family is instantiated for each entry; the C ABI reports any
// other shape as unsupported.
#pragma once

#define CGTP_CONFIGS(X) \
  X(0, 0, 0)            \
  X(1, 1, 1)            \
  X(1, 2, 1)            \
  X(2, 2, 2)            \
  X(2, 4, 2)            \
  X(3, 3, 3)
