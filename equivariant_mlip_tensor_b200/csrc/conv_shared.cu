// Convolution with one weight row per edge shared by every path (path
// stride 0: W_e[p][u] = w_e[u]), forward and backward, for sm_100a:
//   out[i][l3,m3][u] = sum_{e in row i} w_e[u] sum_p sum_{m1,m2} C^p x[j][l1,m1][u] Y_e[l2,m2]
//   grad_w[e][u]     = sum_p (the per-path weight gradient of the channelwise convolution)
// ("Tensor Decomposition Networks ...", reply to reviewer oXft: weights shared
// across paths).  The kernels are those of conv_fwd.cu and conv_bwd.cu with
// one staged weight row per edge instead of one per path, built as separate
// variants in their own translation unit; the backward's chunks run in plain
// stream order because each adds onto the previous chunk's gradient rows.
#include "common.cuh"

namespace cgtp {
CGTP_DEFINE_CONSTANT_TABLES()
}  // namespace cgtp

#include "conv_common.cuh"
#include "vec2.cuh"
#include "sh.cuh"

namespace cgtp {
namespace {

// Warps per block, whether the grid is persistent (one wave that loops over
// the work items) or one group of lanes per item, and the shared-memory
// budget per warp (floats) that sizes the edge batch.  One-warp blocks over
// one item each let the block scheduler balance rows of unequal degree: an
// SM takes a new row as soon as any of its warps finishes one.
#ifndef CGTP_FWD_WARPS
#define CGTP_FWD_WARPS 1
#endif
#ifndef CGTP_FWD_PERSISTENT
#define CGTP_FWD_PERSISTENT 0
#endif
#ifndef CGTP_FWD_BATCH_FLOATS
#define CGTP_FWD_BATCH_FLOATS 12288
#endif
#ifndef CGTP_FWD_MAX_BATCH
#define CGTP_FWD_MAX_BATCH 16
#endif
#ifndef CGTP_FWD_MINB
#define CGTP_FWD_MINB 1
#endif
constexpr int kFwdThreads = 32 * CGTP_FWD_WARPS;
#if CGTP_FWD_MINB > 0
#define CGTP_FWD_BOUNDS __launch_bounds__(kFwdThreads, CGTP_FWD_MINB)
#else
#define CGTP_FWD_BOUNDS __launch_bounds__(kFwdThreads)
#endif
#ifndef CGTP_FWD_VEC
#define CGTP_FWD_VEC 4
#endif
constexpr int kFwdVec = CGTP_FWD_VEC;  // channels per lane

// Stage x rows through the cp.async pipeline (1) or gather them with cached
// loads after an L2 prefetch (0).
#ifndef CGTP_FWD_STAGE_X
#define CGTP_FWD_STAGE_X 1
#endif
constexpr bool kStageX = CGTP_FWD_STAGE_X != 0;

// One launch over all paths while their unrolled code per edge and lane stays
// within CGTP_FWD_SINGLE_MAX instructions; otherwise one launch per chunk of
// paths with one l3, each within CGTP_FWD_BUDGET (the instruction cache).
#ifndef CGTP_FWD_SINGLE_MAX
#define CGTP_FWD_SINGLE_MAX 1600
#endif
#ifndef CGTP_FWD_BUDGET
#define CGTP_FWD_BUDGET 1100
#endif

// One edge: acc[m3][c] += sum_p W[p][c] sum_m1 T[p][m1][m3] x[l1,m1][c] for the group's paths.
template <class PS, class GR>
__device__ __forceinline__ void fwd_edge(const float* __restrict__ T, const float* __restrict__ stage, int rowf,
                                         const float* __restrict__ xg, int mult,
                                         float (&acc)[GR::NOWN][kFwdVec]) {
  float xr[GR::NROW][kFwdVec];
#pragma unroll
  for (int r = 0; r < GR::NROW; ++r) {
    if constexpr (kStageX) VecIO<kFwdVec>::lds(xr[r], stage + (1 + r) * rowf);
    else VecIO<kFwdVec>::ld(xr[r], xg + r * mult);
  }
  static_for<0, GR::NP>([&](auto Kc) {
    constexpr int K = decltype(Kc)::value;
    constexpr int P = GR::D.path[K];
    constexpr int l1 = PS::D.l1[P], l3 = PS::D.l3[P];
    constexpr int tc = PS::D.tcount[P], tb = GR::D.lt[K];
    float wv[kFwdVec];
    VecIO<kFwdVec>::lds(wv, stage);  // the one weight row, shared by every path
    constexpr int o3 = l3 * l3 - GR::OWN0;  // first own row of this path's output block
    if constexpr (2 * l3 + 1 <= 2 * l1 + 1) {
      // t[m3] = sum_m1 T x[m1], then out[m3] += W t[m3]
      float t[2 * l3 + 1][kFwdVec];
#pragma unroll
      for (int m3 = 0; m3 < 2 * l3 + 1; ++m3)
#pragma unroll
        for (int c = 0; c < kFwdVec; ++c) t[m3][c] = 0.f;
      static_for<0, (tc + 3) / 4>([&](auto Qc) {
        constexpr int q = decltype(Qc)::value;
        const float4 v4 = *reinterpret_cast<const float4*>(T + tb + 4 * q);
        const float tv4[4] = {v4.x, v4.y, v4.z, v4.w};
        static_for<0, 4>([&](auto Rc) {
          constexpr int k = 4 * q + decltype(Rc)::value;
          if constexpr (k < tc) {
            constexpr int m1 = PS::t_entry_m1(P, k), m3 = PS::t_entry_m3(P, k);
            constexpr int rx = l1 * l1 + l1 + m1 - GR::D.rlo;
            axpy<kFwdVec>(t[m3 + l3], tv4[decltype(Rc)::value], xr[rx]);
          }
        });
      });
#pragma unroll
      for (int m3 = 0; m3 < 2 * l3 + 1; ++m3) vfma<kFwdVec>(acc[o3 + m3], wv, t[m3]);
    } else {
      // xw[m1] = W x[m1], then out[m3] += sum_m1 T xw[m1]
      float xw[2 * l1 + 1][kFwdVec];
#pragma unroll
      for (int m1 = 0; m1 < 2 * l1 + 1; ++m1) vmul<kFwdVec>(xw[m1], wv, xr[l1 * l1 + m1 - GR::D.rlo]);
      static_for<0, (tc + 3) / 4>([&](auto Qc) {
        constexpr int q = decltype(Qc)::value;
        const float4 v4 = *reinterpret_cast<const float4*>(T + tb + 4 * q);
        const float tv4[4] = {v4.x, v4.y, v4.z, v4.w};
        static_for<0, 4>([&](auto Rc) {
          constexpr int k = 4 * q + decltype(Rc)::value;
          if constexpr (k < tc) {
            constexpr int m1 = PS::t_entry_m1(P, k), m3 = PS::t_entry_m3(P, k);
            axpy<kFwdVec>(acc[o3 + m3 + l3], tv4[decltype(Rc)::value], xw[m1 + l1]);
          }
        });
      });
    }
  });
}

// GR: the launch's paths (all of them, or one chunk of one l3 block).  A
// chunk that continues an l3 block another chunk of the call started adds
// onto that chunk's rows (GR::FIRST false).
template <class PS, class GR, int KMULT>
__global__ void CGTP_FWD_BOUNDS
conv_fwd_kernel(ConvFwdArgs a, int lg_G_rt, int S_rt, int BT) {
  // KMULT > 0: the multiplicity is a compile-time multiple of 32 lanes x 4
  // channels, so every row offset below folds into an immediate.
  const int mult = KMULT ? KMULT : a.mult;
  const int lg_G = KMULT ? 5 : lg_G_rt;
  const int S = KMULT ? KMULT / (32 * kFwdVec) : S_rt;
  constexpr int NI = PS::NI, NO = PS::NO, NS = PS::NS, NT = GR::NT;
  constexpr int NROWS = 1 + (kStageX ? GR::NROW : 0);
  extern __shared__ float4 smem_f4[];
  float* smem = reinterpret_cast<float*>(smem_f4);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int G = 1 << lg_G, gpw = 32 >> lg_G;
  const int grp = lane >> lg_G, gl = lane & (G - 1);
  const int rowf = G * kFwdVec;                    // floats per staged row
  const int stage_floats = NROWS * rowf;
  const int group_floats = BT * NT + 2 * stage_floats + ((BT + 3) & ~3);
  float* Tg = smem + (warp * gpw + grp) * group_floats;
  float* St = Tg + BT * NT;                        // two pipeline stages
  int* Jg = reinterpret_cast<int*>(St + 2 * stage_floats);

  // The next chunk of this call may start on SMs this grid leaves idle (see
  // the launcher: chunks write disjoint rows unless one continues another).
  grid_dependents_launch();
  const long long n_items = (long long)a.n_nodes * S;
  const long long warps_total = (long long)gridDim.x * (kFwdThreads / 32);
  for (long long base = ((long long)blockIdx.x * (kFwdThreads / 32) + warp) * gpw; base < n_items;
       base += warps_total * gpw) {
    const long long item = base + grp;
    const bool active = item < n_items;
    const int node = active ? int(item / S) : 0;
    const int slice = active ? int(item % S) : 0;
    const int c0 = (slice * G + gl) * kFwdVec;
    int e0 = 0, e1 = 0;
    if (active) {
      e0 = __ldg(a.row_ptr + node);
      e1 = __ldg(a.row_ptr + node + 1);
    }
    const int maxdeg = __reduce_max_sync(0xffffffffu, e1 - e0);
    float acc[GR::NOWN][kFwdVec];
#pragma unroll
    for (int r = 0; r < GR::NOWN; ++r)
#pragma unroll
      for (int c = 0; c < kFwdVec; ++c) acc[r][c] = 0.f;

    // copies of edge slot k of the current batch into stage s (this lane's channels only)
    auto issue = [&](int b0, int k, int s) {
      const int e = e0 + b0 + k;
      if (!(active && e < e1)) return;
      float* dst = St + s * stage_floats + gl * kFwdVec;
      VecIO<kFwdVec>::cp_async(dst, a.w + (long long)e * mult + c0);
      if constexpr (kStageX) {
        constexpr int rlo = GR::D.rlo;
        const float* xrow = a.x + ((long long)Jg[k] * NI + rlo) * mult + c0;
#pragma unroll
        for (int r = 0; r < GR::NROW; ++r) VecIO<kFwdVec>::cp_async(dst + (1 + r) * rowf, xrow + r * mult);
      }
    };

    for (int b0 = 0; b0 < maxdeg; b0 += BT) {
      // sources of every slot, then the first slot's copies, so that they fly
      // while the T matrices of the batch are computed
      for (int k = gl; k < BT; k += G) {
        const int e = e0 + b0 + k;
        if (active && e < e1) {
          const int j = __ldg(a.col + e);
          if constexpr (!kStageX) {
            constexpr int rlo = GR::D.rlo;
            prefetch_l2(a.x + ((long long)j * NI + rlo) * mult, (unsigned)(GR::NROW * mult * 4));
          }
          Jg[k] = j;
        }
      }
      __syncwarp();
      const int nb = min(BT, maxdeg - b0);
      issue(b0, 0, 0);
      cp_async_commit();
      for (int k = gl; k < BT; k += G) {
        const int e = e0 + b0 + k;
        if (active && e < e1) {
          float Y[NS];
          edge_sh<PS::LS>(a.sh, a.edge_vec, e, Y);
          compute_T_grp<PS, GR>(Y, Tg + k * NT);
        }
      }
      __syncwarp();
      for (int k = 0; k < nb; ++k) {
        if (k + 1 < nb) issue(b0, k + 1, (k + 1) & 1);
        cp_async_commit();
        cp_async_wait<1>();  // this lane's copies of edge k have landed
        if (active && e0 + b0 + k < e1) {
          constexpr int rlo = GR::D.rlo;
          fwd_edge<PS, GR>(Tg + k * NT, St + (k & 1) * stage_floats + gl * kFwdVec, rowf,
                           a.x + ((long long)Jg[k] * NI + rlo) * mult + c0, mult, acc);
        }
      }
      __syncwarp();
    }
    if (active) {
      if (!GR::FIRST || a.accumulate) {
        // rows of an l3 block that the preceding launch wrote (wait for it),
        // or the caller's values to add onto
        if constexpr (!GR::FIRST) grid_dependency_wait();
#pragma unroll
        for (int r = 0; r < GR::NOWN; ++r) {
          float prev[kFwdVec];
          VecIO<kFwdVec>::ld(prev, a.out + ((long long)node * NO + GR::OWN0 + r) * mult + c0);
#pragma unroll
          for (int c = 0; c < kFwdVec; ++c) acc[r][c] += prev[c];
        }
      }
#pragma unroll
      for (int r = 0; r < GR::NOWN; ++r)
        VecIO<kFwdVec>::st(a.out + ((long long)node * NO + GR::OWN0 + r) * mult + c0, acc[r]);
    }
  }
}

template <class PS, class GR>
cudaError_t launch_fwd_group(const ConvFwdArgs& a, int num_sms, bool pdl, cudaStream_t stream) {
  int G, lg_G, S;
  lane_geometry(a.mult, kFwdVec, G, lg_G, S);
  const int gpw = 32 / G;
  const int stage_floats = (1 + (kStageX ? GR::NROW : 0)) * G * kFwdVec;
  const int BT = pick_batch(gpw, GR::NT, stage_floats, CGTP_FWD_BATCH_FLOATS, CGTP_FWD_MAX_BATCH);
  const int group_floats = BT * GR::NT + 2 * stage_floats + ((BT + 3) & ~3);
  const size_t smem = sizeof(float) * (size_t)group_floats * gpw * (kFwdThreads / 32);
  auto kern = a.mult == 128 ? conv_fwd_kernel<PS, GR, 128> : conv_fwd_kernel<PS, GR, 0>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const long long items = (long long)a.n_nodes * S;
  const long long groups_per_block = (long long)gpw * (kFwdThreads / 32);
  long long blocks = (items + groups_per_block - 1) / groups_per_block;
  long long cap = 0x7fffffffLL;  // the kernel loops over items beyond the grid
  if (CGTP_FWD_PERSISTENT) {
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFwdThreads, smem);
    if (err != cudaSuccess) return err;
    cap = (long long)num_sms * (per_sm < 1 ? 1 : per_sm);
  }
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return launch_kernel(kern, dim3((unsigned)blocks), dim3(kFwdThreads), smem, stream, pdl, a, lg_G, S, BT);
}

// Unrolled instructions per edge and lane of all paths in one launch.
template <class PS>
constexpr int fwd_all_cost() {
  int c = 0;
  for (int p = 0; p < PS::D.np; ++p) c += path_cost<PS>(p, kByL3, kFwdVec, false);
  return c;
}

template <class PS>
using FwdPlan = Plan<PS, kByL3, kFwdVec, false, CGTP_FWD_BUDGET>;

// Output blocks l3 that no path reaches are zero.
template <class PS>
cudaError_t zero_unreached_out(const ConvFwdArgs& a, cudaStream_t stream) {
  cudaError_t err = cudaSuccess;
  static_for_host<0, PS::LO + 1>([&](auto Lc) {
    constexpr int l3 = decltype(Lc)::value;
    constexpr bool reached = [] {
      for (int p = 0; p < PS::D.np; ++p)
        if (PS::D.l3[p] == l3) return true;
      return false;
    }();
    if (!reached && err == cudaSuccess)
      err = cudaMemset2DAsync(a.out + (size_t)l3 * l3 * a.mult, sizeof(float) * PS::NO * a.mult, 0,
                              sizeof(float) * (2 * l3 + 1) * a.mult, a.n_nodes, stream);
  });
  return err;
}

}  // namespace

template <int LI, int LS, int LO>
cudaError_t launch_conv_fwd_shared(const ConvFwdArgs& a, int num_sms, cudaStream_t stream) {
  using PS = PathSet<LI, LS, LO>;
  if constexpr (fwd_all_cost<PS>() <= CGTP_FWD_SINGLE_MAX) {
    // all paths in one launch (it writes every output row, reached or not)
    return launch_fwd_group<PS, Grp<PS, kAll, 0>>(a, num_sms, false, stream);
  } else {
    cudaError_t err = a.accumulate ? cudaSuccess : zero_unreached_out<PS>(a, stream);
    static_for_host<0, FwdPlan<PS>::N>([&](auto Cc) {
      constexpr int CH = decltype(Cc)::value;
      // every chunk but the call's first may overlap the one before it
      if (err == cudaSuccess)
        err = launch_fwd_group<PS, ChunkGrp<PS, FwdPlan<PS>, CH, kByL3>>(a, num_sms, CH > 0, stream);
    });
    return err;
  }
}

// One translation unit per shape (the build passes CGTP_CFG_LI/LS/LO).
template cudaError_t launch_conv_fwd_shared<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(const ConvFwdArgs&, int,
                                                                                cudaStream_t);

}  // namespace cgtp

namespace cgtp {

namespace {

// Warps per block, persistent grid or one group of lanes per item, and the
// shared-memory budget per warp (floats) that sizes the edge batch (as in
// the forward: one-warp blocks let the block scheduler balance the rows).
#ifndef CGTP_BWD_WARPS
#define CGTP_BWD_WARPS 1
#endif
#ifndef CGTP_BWD_PERSISTENT
#define CGTP_BWD_PERSISTENT 0
#endif
#ifndef CGTP_BWD_BATCH_FLOATS
#define CGTP_BWD_BATCH_FLOATS 6144
#endif
#ifndef CGTP_BWD_MAX_BATCH
#define CGTP_BWD_MAX_BATCH 16
#endif
#ifndef CGTP_BWD_MINB
#define CGTP_BWD_MINB 0
#endif
constexpr int kBwdThreads = 32 * CGTP_BWD_WARPS;
#if CGTP_BWD_MINB > 0
#define CGTP_BWD_BOUNDS __launch_bounds__(kBwdThreads, CGTP_BWD_MINB)
#else
#define CGTP_BWD_BOUNDS __launch_bounds__(kBwdThreads)
#endif

template <class PS, class GR>
constexpr unsigned touched_sh_mask() {
  unsigned m = 0;
  for (int k = 0; k < GR::D.n; ++k) {
    const int l2 = PS::D.l2[GR::D.path[k]];
    for (int b = l2 * l2; b < (l2 + 1) * (l2 + 1); ++b) m |= 1u << b;
  }
  return m;
}

// One edge of the CSC row, the paths of one group (l1 = GR's value).  Per
// path, with h[m1] = sum_m3 T[m1][m3] g[m3] (one pass over the structural
// nonzeros of T):
//   grad_x[m1] += W h[m1],   grad_W = sum_m1 x[m1] h[m1],
// and, for grad_Y, the channel sums sum_u W x[m1] g[m3] of every T entry
// contracted with the CG coefficients.  Paths are visited in (l2, ...) order
// so that only one l2 block of the grad_Y partial is live at a time; each
// finished block goes to this lane's column of the shared reduction buffer
// (gyrow, row stride rs).  The edge's weight rows and its destination's output-gradient
// rows come from this lane's pipeline stage.
template <class PS, class GR, int VEC, bool NEED_GY>
__device__ __forceinline__ void bwd_edge(const float* __restrict__ T, const float* __restrict__ stage, int rowf,
                                         const float (&xr)[GR::NOWN][VEC], float* __restrict__ gwrow, bool acc, int mult,
                                         float (&gx)[GR::NOWN][VEC], float* __restrict__ gyrow, int rs) {
  float gy[PS::NS];
  float gws[VEC];  // grad of the shared weight row: sum over this chunk's paths
#pragma unroll
  for (int c = 0; c < VEC; ++c) gws[c] = 0.f;
  static_for<0, GR::NP>([&](auto Kc) {
    constexpr int K = decltype(Kc)::value;
    constexpr int P = GR::D.path[K];
    constexpr int l1 = PS::D.l1[P], l2 = PS::D.l2[P], l3 = PS::D.l3[P];
    constexpr int tb = GR::D.lt[K], tc = PS::D.tcount[P];
    constexpr int g0 = 1 + l3 * l3 - GR::D.rlo;  // staged row of grad_out[l3, m3 = -l3]
    if constexpr (NEED_GY && GR::D.first_l2[K]) {
#pragma unroll
      for (int m2 = 0; m2 < 2 * l2 + 1; ++m2) gy[l2 * l2 + m2] = 0.f;
    }
    float wv[VEC];
    VecIO<VEC>::lds(wv, stage);  // the one weight row, shared by every path
    float gv[2 * l3 + 1][VEC], h[2 * l1 + 1][VEC];
#pragma unroll
    for (int m3 = 0; m3 < 2 * l3 + 1; ++m3) VecIO<VEC>::lds(gv[m3], stage + (g0 + m3) * rowf);
#pragma unroll
    for (int m1 = 0; m1 < 2 * l1 + 1; ++m1)
#pragma unroll
      for (int c = 0; c < VEC; ++c) h[m1][c] = 0.f;
    float xw[2 * l1 + 1][VEC];  // W x, for the grad_Y channel sums
    if constexpr (NEED_GY) {
#pragma unroll
      for (int m1 = 0; m1 < 2 * l1 + 1; ++m1) vmul<VEC>(xw[m1], wv, xr[m1]);
    }
    static_for<0, (tc + 3) / 4>([&](auto Qc) {
      constexpr int q = decltype(Qc)::value;
      const float4 v4 = *reinterpret_cast<const float4*>(T + tb + 4 * q);
      const float tv4[4] = {v4.x, v4.y, v4.z, v4.w};
      static_for<0, 4>([&](auto Rc) {
        constexpr int k = 4 * q + decltype(Rc)::value;
        if constexpr (k < tc) {
          constexpr int m1 = PS::t_entry_m1(P, k), m3 = PS::t_entry_m3(P, k);
          const float tv = tv4[decltype(Rc)::value];
          axpy<VEC>(h[m1 + l1], tv, gv[m3 + l3]);
          if constexpr (NEED_GY) {
            const float av = vdot<VEC>(xw[m1 + l1], gv[m3 + l3]);
            static_for<0, 2 * l2 + 1>([&](auto M2c) {
              constexpr int m2 = decltype(M2c)::value - l2;
              if constexpr (cg_allowed(l1, l2, l3, m1, m2, m3)) {
                gy[l2 * l2 + l2 + m2] = fmaf(c_cg[table_index(l1, l2, l3, m1, m2, m3)], av, gy[l2 * l2 + l2 + m2]);
              }
            });
          }
        }
      });
    });
#pragma unroll
    for (int m1 = 0; m1 < 2 * l1 + 1; ++m1) {
      vfma<VEC>(gx[m1], wv, h[m1]);
      vfma<VEC>(gws, xr[m1], h[m1]);
    }
    if constexpr (NEED_GY && GR::D.last_l2[K]) {
#pragma unroll
      for (int m2 = 0; m2 < 2 * l2 + 1; ++m2) gyrow[(l2 * l2 + m2) * rs] = gy[l2 * l2 + m2];
    }
  });
  if (gwrow != nullptr) {
    if (acc) {  // a preceding chunk of this call wrote the row: add onto it
      float prev[VEC];
      VecIO<VEC>::ld(prev, gwrow);
#pragma unroll
      for (int c = 0; c < VEC; ++c) gws[c] += prev[c];
    }
    VecIO<VEC>::st_stream(gwrow, gws);
  }
}

// Unrolled instructions per edge and lane allowed in one backward launch.
#ifndef CGTP_BWD_BUDGET
#define CGTP_BWD_BUDGET 1100
#endif
#ifndef CGTP_BWD_BUDGET_L3
#define CGTP_BWD_BUDGET_L3 800  // l = 3 chunks carry more registers per path
#endif
template <class PS>
constexpr int bwd_budget() {
  return PS::LI >= 3 || PS::LO >= 3 ? CGTP_BWD_BUDGET_L3 : CGTP_BWD_BUDGET;
}

template <class PS, int VEC, bool NEED_GY>
using BwdPlan = Plan<PS, kByL1, VEC, NEED_GY, bwd_budget<PS>()>;

// One launch per chunk (paths of one l1 block): grad_x rows of that block
// (written by the block's first chunk, accumulated by the others), grad_W
// of the chunk's paths and a partial grad_Y over them.
// EXT: the double backward's variant (per-edge harmonics given by the caller,
// results added onto the outputs); the plain variant compiles without either.
template <class PS, int VEC, bool NEED_GY, int CH, int KMULT, bool EXT>
__global__ void CGTP_BWD_BOUNDS
conv_bwd_kernel(ConvBwdArgs a, int lg_G_rt, int S_rt, int BT, int slice_base_rt) {
  // KMULT > 0: the multiplicity is a compile-time multiple of 32 lanes x VEC
  // channels, so every row offset below folds into an immediate.
  const int mult = KMULT ? KMULT : a.mult;
  const int lg_G = KMULT ? 5 : lg_G_rt;
  const int S = KMULT ? KMULT / (32 * VEC) : S_rt;
  const int slice_base = KMULT ? CH * S : slice_base_rt;
  using GR = ChunkGrp<PS, BwdPlan<PS, VEC, NEED_GY>, CH, kByL1>;
  constexpr int L1 = GR::KEY;
  constexpr int NI = PS::NI, NO = PS::NO, NS = PS::NS, NR = GR::NOWN, NT = GR::NT;
  constexpr int NROWS = 1 + GR::NROW;
  constexpr unsigned GY_MASK = touched_sh_mask<PS, GR>();  // harmonics this chunk's paths reach
  extern __shared__ float4 smem_f4[];
  float* smem = reinterpret_cast<float*>(smem_f4);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int G = 1 << lg_G, gpw = 32 >> lg_G;
  const int grp = lane >> lg_G, gl = lane & (G - 1);
  const int rowf = G * VEC;
  const int stage_floats = NROWS * rowf;
  const int group_floats = BT * NT + 2 * stage_floats + 2 * ((BT + 3) & ~3);
  float* Tg = smem + (warp * gpw + grp) * group_floats;
  float* St = Tg + BT * NT;
  int* Eg = reinterpret_cast<int*>(St + 2 * stage_floats);
  int* Ig = Eg + ((BT + 3) & ~3);
  // grad_Y reduction buffer, per group of lanes: NS rows (one per harmonic)
  // of G lane partials, row stride rs = G + 4 (float4 aligned, and rows read
  // by the 8 lanes of one 128-bit access phase fall in distinct banks)
  const int rs = G + 4;
  float* red = smem + (kBwdThreads / 32) * gpw * group_floats + (warp * gpw + grp) * NS * rs;

  // The next chunk of this call may start on SMs this grid leaves idle: no
  // chunk reads what another writes, except a chunk that adds onto an
  // earlier chunk's grad_x rows, and that one waits for it below.
  grid_dependents_launch();
  const long long n_items = (long long)a.n_nodes * S;
  const long long warps_total = (long long)gridDim.x * (kBwdThreads / 32);
  for (long long base = ((long long)blockIdx.x * (kBwdThreads / 32) + warp) * gpw; base < n_items;
       base += warps_total * gpw) {
    const long long item = base + grp;
    const bool active = item < n_items;
    const long long node = active ? item / S : 0;
    const int slice = active ? int(item % S) : 0;
    const int c0 = (slice * G + gl) * VEC;
    int k0 = 0, k1 = 0;
    if (active) {
      k0 = __ldg(a.csc_ptr + node);
      k1 = __ldg(a.csc_ptr + node + 1);
    }
    const int maxdeg = __reduce_max_sync(0xffffffffu, k1 - k0);
    float xr[NR][VEC], gx[NR][VEC];
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      if (active) VecIO<VEC>::ld(xr[r], a.x + (node * NI + L1 * L1 + r) * mult + c0);
      else {
#pragma unroll
        for (int c = 0; c < VEC; ++c) xr[r][c] = 0.f;
      }
#pragma unroll
      for (int c = 0; c < VEC; ++c) gx[r][c] = 0.f;
    }

    // copies of edge slot k of the current batch into stage s (this lane's channels only)
    auto issue = [&](int b0, int k, int s) {
      if (!(active && k0 + b0 + k < k1)) return;
      float* dst = St + s * stage_floats + gl * VEC;
      VecIO<VEC>::cp_async(dst, a.w + (long long)Eg[k] * mult + c0);
      constexpr int rlo = GR::D.rlo;
      const float* grow = a.grad_out + ((long long)Ig[k] * NO + rlo) * mult + c0;
#pragma unroll
      for (int r = 0; r < GR::NROW; ++r) VecIO<VEC>::cp_async(dst + (1 + r) * rowf, grow + r * mult);
    };

    for (int b0 = 0; b0 < maxdeg; b0 += BT) {
      for (int k = gl; k < BT; k += G) {
        const int kk = k0 + b0 + k;
        if (active && kk < k1) {
          const int e = __ldg(a.csc_edge + kk);
          float Y[NS];
          edge_sh<PS::LS>(EXT ? a.sh : nullptr, a.edge_vec, e, Y);
          compute_T_grp<PS, GR>(Y, Tg + k * NT);
          Eg[k] = e;
          Ig[k] = __ldg(a.csc_dst + kk);
        }
      }
      __syncwarp();
      const int nb = min(BT, maxdeg - b0);
      issue(b0, 0, 0);
      cp_async_commit();
      for (int k = 0; k < nb; ++k) {
        if (k + 1 < nb) issue(b0, k + 1, (k + 1) & 1);
        cp_async_commit();
        cp_async_wait<1>();  // this lane's copies of edge k have landed
        const bool valid = active && (k0 + b0 + k) < k1;
        int e = 0;
        if (valid) {
          e = Eg[k];
          bwd_edge<PS, GR, VEC, NEED_GY>(Tg + k * NT, St + (k & 1) * stage_floats + gl * VEC, rowf, xr,
                                         a.grad_w ? a.grad_w + (long long)e * mult + c0 : nullptr,
                                         CH > 0 || (EXT && a.accumulate != 0), mult, gx, red + gl, rs);
        }
        if constexpr (NEED_GY) {
          __syncwarp();
          if (valid) {
            float* dst = a.grad_sh + ((long long)(slice_base + slice) * a.n_edges + e) * NS;
            for (int b = gl; b < NS; b += G) {  // column sums; harmonics the chunk never reaches get 0
              float v = 0.f;
              if ((GY_MASK >> b) & 1u) {
                const float* row = red + b * rs;
                if (G % 4 == 0) {
                  float4 s4 = make_float4(0.f, 0.f, 0.f, 0.f);
                  for (int r = 0; r < G; r += 4) {
                    const float4 q4 = *reinterpret_cast<const float4*>(row + r);
                    s4.x += q4.x;
                    s4.y += q4.y;
                    s4.z += q4.z;
                    s4.w += q4.w;
                  }
                  v = (s4.x + s4.y) + (s4.z + s4.w);
                } else {
                  for (int r = 0; r < G; ++r) v += row[r];
                }
              }
              dst[b] = v;
            }
          }
          __syncwarp();
        }
      }
      __syncwarp();
    }
    if (active && a.grad_x != nullptr) {
      if (!GR::FIRST || (EXT && a.accumulate)) {
        // rows of an l1 block that an earlier chunk of this call wrote (wait
        // for that grid, the preceding launch), or the caller's values
        if constexpr (!GR::FIRST) grid_dependency_wait();
#pragma unroll
        for (int r = 0; r < NR; ++r) {
          float prev[VEC];
          VecIO<VEC>::ld(prev, a.grad_x + (node * NI + L1 * L1 + r) * mult + c0);
#pragma unroll
          for (int c = 0; c < VEC; ++c) gx[r][c] += prev[c];
        }
      }
#pragma unroll
      for (int r = 0; r < NR; ++r) VecIO<VEC>::st(a.grad_x + (node * NI + L1 * L1 + r) * mult + c0, gx[r]);
    }
  }
}

// grad_edge_vec[e] (= or +=) (dY_e/dr_e)^T sum_s grad_sh[s][e]
template <int LS>
__global__ void sh_backward_kernel(int n_edges, int S, const float* __restrict__ edge_vec,
                                   const float* __restrict__ grad_sh, float* __restrict__ grad_edge_vec, int add) {
  constexpr int NS = (LS + 1) * (LS + 1);
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n_edges;
       e += (long long)gridDim.x * blockDim.x) {
    float g[NS];
#pragma unroll
    for (int b = 0; b < NS; ++b) g[b] = 0.f;
    for (int s = 0; s < S; ++s) {
      const float* src = grad_sh + ((long long)s * n_edges + e) * NS;
#pragma unroll
      for (int b = 0; b < NS; ++b) g[b] += src[b];
    }
    Dual3 Y[NS];
    sh_grad_of_vec<LS>(edge_vec[3 * e], edge_vec[3 * e + 1], edge_vec[3 * e + 2], Y);
    float d0 = 0.f, d1 = 0.f, d2 = 0.f;
#pragma unroll
    for (int b = 0; b < NS; ++b) {
      d0 = fmaf(g[b], Y[b].d0, d0);
      d1 = fmaf(g[b], Y[b].d1, d1);
      d2 = fmaf(g[b], Y[b].d2, d2);
    }
    if (add) {
      d0 += grad_edge_vec[3 * e];
      d1 += grad_edge_vec[3 * e + 1];
      d2 += grad_edge_vec[3 * e + 2];
    }
    grad_edge_vec[3 * e] = d0;
    grad_edge_vec[3 * e + 1] = d1;
    grad_edge_vec[3 * e + 2] = d2;
  }
}

// grad_edge_vec[e] (= or +=) sum_b G_b (d2Y_b/dr2) q_e with G = sum_s grad_sh[s][e]:
// the second-order term of the double backward (q = the cotangent of grad_edge_vec).
template <int LS>
__global__ void sh_backward_hess_kernel(int n_edges, int S, const float* __restrict__ edge_vec,
                                        const float* __restrict__ grad_sh, const float* __restrict__ q,
                                        float* __restrict__ grad_edge_vec, int add) {
  constexpr int NS = (LS + 1) * (LS + 1);
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n_edges;
       e += (long long)gridDim.x * blockDim.x) {
    float g[NS];
#pragma unroll
    for (int b = 0; b < NS; ++b) g[b] = 0.f;
    for (int s = 0; s < S; ++s) {
      const float* src = grad_sh + ((long long)s * n_edges + e) * NS;
#pragma unroll
      for (int b = 0; b < NS; ++b) g[b] += src[b];
    }
    HDual Y[NS];
    sh_hess_of_vec<LS>(edge_vec[3 * e], edge_vec[3 * e + 1], edge_vec[3 * e + 2], q[3 * e], q[3 * e + 1],
                       q[3 * e + 2], Y);
    float d0 = 0.f, d1 = 0.f, d2 = 0.f;
#pragma unroll
    for (int b = 0; b < NS; ++b) {
      d0 = fmaf(g[b], Y[b].d0.e, d0);
      d1 = fmaf(g[b], Y[b].d1.e, d1);
      d2 = fmaf(g[b], Y[b].d2.e, d2);
    }
    if (add) {
      d0 += grad_edge_vec[3 * e];
      d1 += grad_edge_vec[3 * e + 1];
      d2 += grad_edge_vec[3 * e + 2];
    }
    grad_edge_vec[3 * e] = d0;
    grad_edge_vec[3 * e + 1] = d1;
    grad_edge_vec[3 * e + 2] = d2;
  }
}

}  // namespace

// Programmatic dependent launch between the chunks of one backward call
// (1) or plain stream order (0).
#ifndef CGTP_BWD_PDL
#define CGTP_BWD_PDL 0  // the chunks add onto each other's weight-gradient rows
#endif

// Channels per lane (float4: measured faster than 2 at every shape with
// one-warp blocks and budgeted chunks).
#ifndef CGTP_BWD_VEC
#define CGTP_BWD_VEC 4
#endif
template <class PS>
constexpr int shared_bwd_vec() {
  return CGTP_BWD_VEC;
}

// channel lanes per group (G) and channel slices (S) of the backward
template <class PS>
void shared_bwd_geometry(int mult, int& G, int& lg_G, int& S) {
  lane_geometry(mult, shared_bwd_vec<PS>(), G, lg_G, S);
}

template <int LI, int LS, int LO>
int shared_bwd_slices(int mult) {
  using PS = PathSet<LI, LS, LO>;
  int G, lg_G, S;
  shared_bwd_geometry<PS>(mult, G, lg_G, S);
  return S * BwdPlan<PS, shared_bwd_vec<PS>(), true>::N;  // one partial grad_Y per (chunk, channel slice)
}

template <class PS, bool NEED_GY, int CH>
cudaError_t shared_bwd_chunk(const ConvBwdArgs& a, int num_sms, cudaStream_t stream) {
  constexpr int VEC = shared_bwd_vec<PS>();
  using GR = ChunkGrp<PS, BwdPlan<PS, VEC, NEED_GY>, CH, kByL1>;
  int G, lg_G, S;
  shared_bwd_geometry<PS>(a.mult, G, lg_G, S);
  const int gpw = 32 / G;
  const int stage_floats = (1 + GR::NROW) * G * VEC;
  const int BT = pick_batch(gpw, GR::NT, stage_floats, CGTP_BWD_BATCH_FLOATS, CGTP_BWD_MAX_BATCH);
  const int group_floats = BT * GR::NT + 2 * stage_floats + 2 * ((BT + 3) & ~3);
  const size_t smem = sizeof(float) * ((size_t)group_floats * gpw * (kBwdThreads / 32) +
                                       (NEED_GY ? (size_t)(kBwdThreads / 32) * gpw * PS::NS * (G + 4) : 0));
  const long long items = (long long)a.n_nodes * S;
  const long long groups_per_block = (long long)gpw * (kBwdThreads / 32);
  const long long blocks = (items + groups_per_block - 1) / groups_per_block;
  if (a.sh != nullptr || a.accumulate) return cudaErrorInvalidValue;
  auto kern = a.mult == 128 ? conv_bwd_kernel<PS, VEC, NEED_GY, CH, 128, false>
                            : conv_bwd_kernel<PS, VEC, NEED_GY, CH, 0, false>;
  cudaError_t e2 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e2 != cudaSuccess) return e2;
  long long cap = 0x7fffffffLL;  // the kernel loops over items beyond the grid
  if (CGTP_BWD_PERSISTENT) {
    int per_sm = 0;
    e2 = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kBwdThreads, smem);
    if (e2 != cudaSuccess) return e2;
    cap = (long long)num_sms * (per_sm < 1 ? 1 : per_sm);
  }
  long long nb = blocks > cap ? cap : blocks;
  if (nb < 1) nb = 1;
  // Every chunk but the call's first may overlap the one before it.
  return launch_kernel(kern, dim3((unsigned)nb), dim3(kBwdThreads), smem, stream, CGTP_BWD_PDL && CH > 0, a, lg_G,
                       S, BT, CH * S);
}

// grad_x blocks that no path reaches (l1 with no path) are zero.
template <class PS>
cudaError_t shared_zero_unreached_grad_x(const ConvBwdArgs& a, cudaStream_t stream) {
  if (a.grad_x == nullptr) return cudaSuccess;
  cudaError_t err = cudaSuccess;
  static_for_host<0, PS::LI + 1>([&](auto Lc) {
    constexpr int l1 = decltype(Lc)::value;
    constexpr bool reached = [] {
      for (int p = 0; p < PS::D.np; ++p)
        if (PS::D.l1[p] == l1) return true;
      return false;
    }();
    if (!reached && err == cudaSuccess)
      err = cudaMemset2DAsync(a.grad_x + (size_t)l1 * l1 * a.mult, sizeof(float) * PS::NI * a.mult, 0,
                              sizeof(float) * (2 * l1 + 1) * a.mult, a.n_nodes, stream);
  });
  return err;
}

template <class PS, bool NEED_GY>
cudaError_t shared_bwd_chunks(const ConvBwdArgs& a, int num_sms, cudaStream_t stream) {
  constexpr int NCH = BwdPlan<PS, shared_bwd_vec<PS>(), NEED_GY>::N;
  cudaError_t err = a.accumulate ? cudaSuccess : shared_zero_unreached_grad_x<PS>(a, stream);
  static_for_host<0, NCH>([&](auto Cc) {
    if (err == cudaSuccess) err = shared_bwd_chunk<PS, NEED_GY, decltype(Cc)::value>(a, num_sms, stream);
  });
  return err;
}

template <int LI, int LS, int LO>
cudaError_t launch_conv_bwd_shared(const ConvBwdArgs& a, int num_sms, cudaStream_t stream) {
  using PS = PathSet<LI, LS, LO>;
  const cudaError_t err = a.grad_edge_vec != nullptr ? shared_bwd_chunks<PS, true>(a, num_sms, stream)
                                                     : shared_bwd_chunks<PS, false>(a, num_sms, stream);
  if (err != cudaSuccess || a.grad_edge_vec == nullptr || a.n_edges == 0) return err;
  const int threads = 256;
  long long nbk = (a.n_edges + threads - 1) / threads;
  if (nbk > (long long)num_sms * 16) nbk = (long long)num_sms * 16;
  const int S = shared_bwd_slices<LI, LS, LO>(a.mult);
  if (a.gr_mode >= 2) {
    if (a.gr_dir == nullptr) return cudaErrorInvalidValue;
    sh_backward_hess_kernel<LS><<<(unsigned)nbk, threads, 0, stream>>>(a.n_edges, S, a.edge_vec, a.grad_sh, a.gr_dir,
                                                                      a.grad_edge_vec, a.gr_mode == 2);
  } else {
    sh_backward_kernel<LS><<<(unsigned)nbk, threads, 0, stream>>>(a.n_edges, S, a.edge_vec, a.grad_sh,
                                                                 a.grad_edge_vec, a.gr_mode == 1);
  }
  return cudaGetLastError();
}

// One translation unit per shape (the build passes CGTP_CFG_LI/LS/LO).
template cudaError_t launch_conv_bwd_shared<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(const ConvBwdArgs&, int,
                                                                         cudaStream_t);
template int shared_bwd_slices<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(int);

}  // namespace cgtp
