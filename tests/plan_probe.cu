// Host-only probe of the backward's compile-time chunk plans: prints each plan
// as one JSON line per (shape, variant) for tests/test_plan_cpu.py.  Built by
// that test with nvcc (no device code is launched).
#include "common.cuh"
namespace cgtp {
CGTP_DEFINE_CONSTANT_TABLES()
// the table uploader lives in the library's C ABI unit, which the probe does not link
int register_table_uploader(cudaError_t (*)(const float*, const float*)) { return 0; }
}  // namespace cgtp
#include "conv_common.cuh"
#include "vec2.cuh"
#include "sh.cuh"
#include "launch.h"
#include "conv_bwd_kernel.cuh"
#include <cstdio>

using namespace cgtp;

template <class PS, class PL>
void emit(const char* variant, int budget) {
  printf("{\"shape\": [%d, %d, %d], \"variant\": \"%s\", \"budget\": %d, \"chunks\": [", PS::LI, PS::LS, PS::LO,
         variant, budget);
  for (int c = 0; c < PL::N; ++c) {
    printf("%s{\"key\": %d, \"key_hi\": %d, \"first_of_key\": %d, \"chain\": %d, \"paths\": [", c ? ", " : "",
           PL::P.key[c], PL::P.key_hi[c], (int)PL::P.first_of_key[c], PL::P.chain[c]);
    for (int k = 0; k < PL::P.count[c]; ++k) {
      const int p = PL::P.order[PL::P.first[c] + k];
      printf("%s[%d, %d, %d, %d]", k ? ", " : "", PS::D.l1[p], PS::D.l2[p], PS::D.l3[p],
             path_cost<PS>(p, kByL1, kBwdVec, true));
    }
    printf("]}");
  }
  printf("], \"chains\": %d, \"n_paths\": %d}\n", PL::CHAINS, PS::D.np);
}

template <int LI, int LS, int LO>
void shape() {
  using PS = PathSet<LI, LS, LO>;
  emit<PS, BwdPlan<PS, true>>("backward", bwd_budget<PS>());
  emit<PS, BwdPlan<PS, true, kVarDD>>("double_backward", dd_bwd_budget<PS>());
}

int main() {
  shape<1, 1, 1>();
  shape<2, 2, 2>();
  shape<2, 4, 2>();
  shape<3, 3, 3>();
  shape<3, 4, 3>();
  shape<2, 3, 2>();
  shape<0, 4, 3>();
  shape<3, 2, 0>();
  return 0;
}
