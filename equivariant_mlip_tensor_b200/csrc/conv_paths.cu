// Per-path stages of the fully connected convolution, for sm_100a: the
// channelwise forward with one block of output rows per path (the messages t
// that the tensor-core mixing consumes) and the channelwise backward with
// one output gradient per path (the gradients that the mixing's transpose
// produces).  The kernels are the convolution kernels of conv_fwd.cu and
// conv_bwd.cu built as separate variants in their own translation unit, so
// that the plain kernels compile exactly as on their own.
#include "common.cuh"

namespace cgtp {
CGTP_DEFINE_CONSTANT_TABLES()
}  // namespace cgtp

#include "conv_common.cuh"
#include "vec2.cuh"
#include "paths_common.cuh"
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
// Programmatic dependent launch between the chunks of one forward call (1)
// or plain stream order (0).
#ifndef CGTP_FWD_PDL
#define CGTP_FWD_PDL 0
#endif
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
    if constexpr (kStageX) VecIO<kFwdVec>::lds(xr[r], stage + (GR::NP + r) * rowf);
    else VecIO<kFwdVec>::ld(xr[r], xg + r * mult);
  }
  static_for<0, GR::NP>([&](auto Kc) {
    constexpr int K = decltype(Kc)::value;
    constexpr int P = GR::D.path[K];
    constexpr int l1 = PS::D.l1[P], l3 = PS::D.l3[P];
    constexpr int tc = PS::D.tcount[P], tb = GR::D.lt[K];
    float wv[kFwdVec];
    VecIO<kFwdVec>::lds(wv, stage + K * rowf);
    // first own row of this path's output: its l3 block, or its own block of
    // 2 l3 + 1 rows when the launch keeps the paths apart
    constexpr int o3 = GR::PERPATH ? K * (2 * l3 + 1) : l3 * l3 - GR::OWN0;
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
  constexpr int NROWS = GR::NP + (kStageX ? GR::NROW : 0);
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
      const float* wrow = a.w + (long long)e * PS::NP * mult + c0;
      static_for<0, GR::NP>([&](auto Kc) {
        constexpr int K = decltype(Kc)::value;
        constexpr int P = GR::D.path[K];
        VecIO<kFwdVec>::cp_async(dst + K * rowf, wrow + P * mult);
      });
      if constexpr (kStageX) {
        constexpr int rlo = GR::D.rlo;
        const float* xrow = a.x + ((long long)Jg[k] * NI + rlo) * mult + c0;
#pragma unroll
        for (int r = 0; r < GR::NROW; ++r) VecIO<kFwdVec>::cp_async(dst + (GR::NP + r) * rowf, xrow + r * mult);
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
    if constexpr (GR::PERPATH) {
      // t[node][m3][rank][u] of this l3 block, rank = the path's place among
      // the block's paths
      if (active) {
        constexpr int n3 = 2 * GR::KEY + 1;
        static_for<0, GR::NP>([&](auto Kc) {
          constexpr int K = decltype(Kc)::value;
#pragma unroll
          for (int m3 = 0; m3 < n3; ++m3)
            VecIO<kFwdVec>::st(a.out + (((long long)node * n3 + m3) * GR::NPK + GR::PL0 + K) * mult + c0,
                               acc[K * n3 + m3]);
        });
      }
    } else if (active) {
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
  // Complete only after the preceding launch of this call: the last grid of a
  // chain of overlapped launches then completes after every earlier one, so
  // work queued behind the chain in the stream sees all of it done.
  grid_dependency_wait();
}

template <class PS, class GR>
cudaError_t launch_fwd_group(const ConvFwdArgs& a, int num_sms, bool pdl, cudaStream_t stream) {
  int G, lg_G, S;
  lane_geometry(a.mult, kFwdVec, G, lg_G, S);
  const int gpw = 32 / G;
  const int stage_floats = (GR::NP + (kStageX ? GR::NROW : 0)) * G * kFwdVec;
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

// Per-path rows (the fully connected convolution's first stage): chunks of
// same-l3 paths that keep one block of 2 l3 + 1 output rows per path, at most
// kPathRowsMax rows per chunk (the accumulators stay in registers).
constexpr int kPathRowsMax = 16;
template <class PS>
using PathPlan = PlanRows<PS, kByL3, kFwdVec, false, CGTP_FWD_BUDGET, kPathRowsMax>;

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
  static constexpr int NPK = key_count();                     // paths with this l3
  static constexpr int PL0 = PL::P.first[CH] - key_first();   // rank of the chunk's first path
};

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

// Per-path messages t (the fully connected convolution's first stage): a.out
// is t, whose block for l3 holds [n_nodes][2 l3 + 1][paths of l3][mult] and
// follows the blocks of smaller l3.
template <int LI, int LS, int LO>
cudaError_t launch_conv_paths(const ConvFwdArgs& a, int num_sms, cudaStream_t stream) {
  using PS = PathSet<LI, LS, LO>;
  using PL = PathPlan<PS>;
  cudaError_t err = cudaSuccess;
  static_for_host<0, PL::N>([&](auto Cc) {
    constexpr int CH = decltype(Cc)::value;
    using GR = PathRowsGrp<PS, PL, CH>;
    size_t off = 0;  // floats before the l3 = KEY block
    for (int c = 0; c < PL::P.n; ++c)
      if (PL::P.key[c] < GR::KEY) off += (size_t)PL::P.count[c] * (2 * PL::P.key[c] + 1);
    ConvFwdArgs b = a;
    b.out = a.out + off * (size_t)a.n_nodes * a.mult;
    b.accumulate = 0;
    // chunks write disjoint rows: all but the first may overlap the one before
    if (err == cudaSuccess) err = launch_fwd_group<PS, GR>(b, num_sms, CGTP_FWD_PDL && CH > 0, stream);
  });
  return err;
}

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

// Per-path output gradients: staged rows of path K of the group start at
// pp_rowoff(K) (each path has its own 2 l3 + 1 rows).
template <class PS, class GR>
constexpr int pp_rowoff(int K) {
  int r = 0;
  for (int k = 0; k < K; ++k) r += 2 * PS::D.l3[GR::D.path[k]] + 1;
  return r;
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
template <class PS, class GR, int VEC, bool NEED_GY, bool PP, bool HX>
__device__ __forceinline__ void bwd_edge(const float* __restrict__ T, const float* __restrict__ stage, int rowf,
                                         const float (&xr)[GR::NOWN][VEC], float* __restrict__ gwrow, bool acc, int mult,
                                         float (&gx)[GR::NOWN][VEC], float* __restrict__ gyrow, int rs) {
  float gy[PS::NS];
  static_for<0, GR::NP>([&](auto Kc) {
    constexpr int K = decltype(Kc)::value;
    constexpr int P = GR::D.path[K];
    constexpr int l1 = PS::D.l1[P], l2 = PS::D.l2[P], l3 = PS::D.l3[P];
    constexpr int tb = GR::D.lt[K], tc = PS::D.tcount[P];
    // staged row of grad_out[l3, m3 = -l3] (of this path's own rows when PP)
    constexpr int g0 = PP ? GR::NP + pp_rowoff<PS, GR>(K) : GR::NP + l3 * l3 - GR::D.rlo;
    if constexpr (NEED_GY && GR::D.first_l2[K]) {
#pragma unroll
      for (int m2 = 0; m2 < 2 * l2 + 1; ++m2) gy[l2 * l2 + m2] = 0.f;
    }
    float wv[VEC];
    VecIO<VEC>::lds(wv, stage + K * rowf);
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
          if constexpr (HX) axpy<VEC>(h[m1 + l1], tv, gv[m3 + l3]);
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
    if constexpr (HX) {
      float gw[VEC];
#pragma unroll
      for (int c = 0; c < VEC; ++c) gw[c] = 0.f;
#pragma unroll
      for (int m1 = 0; m1 < 2 * l1 + 1; ++m1) {
        vfma<VEC>(gx[m1], wv, h[m1]);
        vfma<VEC>(gw, xr[m1], h[m1]);
      }
      if (gwrow != nullptr) {
        if (acc) {
          float prev[VEC];
          VecIO<VEC>::ld(prev, gwrow + P * mult);
#pragma unroll
          for (int c = 0; c < VEC; ++c) gw[c] += prev[c];
        }
        VecIO<VEC>::st_stream(gwrow + P * mult, gw);
      }
    }
    if constexpr (NEED_GY && GR::D.last_l2[K]) {
#pragma unroll
      for (int m2 = 0; m2 < 2 * l2 + 1; ++m2) gyrow[(l2 * l2 + m2) * rs] = gy[l2 * l2 + m2];
    }
  });
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
// PP: grad_out is the per-path message layout of the fully connected
// convolution (each path reads its own rows).
// HX = false: only the harmonic gradient (no grad_x, no grad_W, and none of
// the T^T g products they need), for passes that want grad_Y alone.
template <class PS, int VEC, bool NEED_GY, int CH, int KMULT, bool EXT, bool PP, bool HX>
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
  constexpr int NG = PP ? pp_rowoff<PS, GR>(GR::NP) : GR::NROW;  // staged gradient rows
  constexpr int NROWS = GR::NP + NG;
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
      const float* wrow = a.w + (long long)Eg[k] * PS::NP * mult + c0;
      static_for<0, GR::NP>([&](auto Kc) {
        constexpr int K = decltype(Kc)::value;
        constexpr int P = GR::D.path[K];
        VecIO<VEC>::cp_async(dst + K * rowf, wrow + P * mult);
      });
      if constexpr (PP) {
        // block l3 of the per-path layout: [node][m3][rank][u]
        static_for<0, GR::NP>([&](auto Kc) {
          constexpr int K = decltype(Kc)::value;
          constexpr int P = GR::D.path[K];
          constexpr int l3 = PS::D.l3[P], n3 = 2 * l3 + 1;
          constexpr int npk = l3_count<PS>(l3), rank = l3_rank<PS>(P), pre = l3_prefix_rows<PS>(l3);
          constexpr int ro = pp_rowoff<PS, GR>(K);
          const float* base = a.grad_out + (long long)a.n_nodes * mult * pre +
                              ((long long)Ig[k] * n3 * npk + rank) * mult + c0;
#pragma unroll
          for (int m3 = 0; m3 < n3; ++m3)
            VecIO<VEC>::cp_async(dst + (GR::NP + ro + m3) * rowf, base + (long long)m3 * npk * mult);
        });
      } else {
        constexpr int rlo = GR::D.rlo;
        const float* grow = a.grad_out + ((long long)Ig[k] * NO + rlo) * mult + c0;
#pragma unroll
        for (int r = 0; r < GR::NROW; ++r) VecIO<VEC>::cp_async(dst + (GR::NP + r) * rowf, grow + r * mult);
      }
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
          bwd_edge<PS, GR, VEC, NEED_GY, PP, HX>(Tg + k * NT, St + (k & 1) * stage_floats + gl * VEC, rowf, xr,
                                         HX && a.grad_w ? a.grad_w + (long long)e * PS::NP * mult + c0 : nullptr,
                                         EXT && a.accumulate != 0, mult, gx, red + gl, rs);
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
    if (HX && active && a.grad_x != nullptr) {
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
  // Complete only after the preceding launch of this call: the last grid of a
  // chain of overlapped launches then completes after every earlier one, so
  // work queued behind the chain in the stream sees all of it done.
  grid_dependency_wait();
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
#define CGTP_BWD_PDL 0
#endif

// Channels per lane (float4: measured faster than 2 at every shape with
// one-warp blocks and budgeted chunks).
#ifndef CGTP_BWD_VEC
#define CGTP_BWD_VEC 4
#endif
template <class PS>
constexpr int paths_bwd_vec() {
  return CGTP_BWD_VEC;
}

// channel lanes per group (G) and channel slices (S) of the backward
template <class PS>
void paths_bwd_geometry(int mult, int& G, int& lg_G, int& S) {
  lane_geometry(mult, paths_bwd_vec<PS>(), G, lg_G, S);
}

template <int LI, int LS, int LO>
int paths_bwd_slices(int mult) {
  using PS = PathSet<LI, LS, LO>;
  int G, lg_G, S;
  paths_bwd_geometry<PS>(mult, G, lg_G, S);
  return S * BwdPlan<PS, paths_bwd_vec<PS>(), true>::N;  // one partial grad_Y per (chunk, channel slice)
}

template <class PS, bool NEED_GY, int CH, bool PP = true, bool HX = true, int KMULT = 0>
cudaError_t paths_bwd_chunk(const ConvBwdArgs& a, int num_sms, cudaStream_t stream) {
  constexpr int VEC = paths_bwd_vec<PS>();
  using GR = ChunkGrp<PS, BwdPlan<PS, VEC, NEED_GY>, CH, kByL1>;
  int G, lg_G, S;
  paths_bwd_geometry<PS>(a.mult, G, lg_G, S);
  const int gpw = 32 / G;
  const int ng = PP ? pp_rowoff<PS, GR>(GR::NP) : GR::NROW;
  const int stage_floats = (GR::NP + ng) * G * VEC;
  const int BT = pick_batch(gpw, GR::NT, stage_floats, CGTP_BWD_BATCH_FLOATS, CGTP_BWD_MAX_BATCH);
  const int group_floats = BT * GR::NT + 2 * stage_floats + 2 * ((BT + 3) & ~3);
  const size_t smem = sizeof(float) * ((size_t)group_floats * gpw * (kBwdThreads / 32) +
                                       (NEED_GY ? (size_t)(kBwdThreads / 32) * gpw * PS::NS * (G + 4) : 0));
  const long long items = (long long)a.n_nodes * S;
  const long long groups_per_block = (long long)gpw * (kBwdThreads / 32);
  const long long blocks = (items + groups_per_block - 1) / groups_per_block;
  if (a.sh != nullptr || a.accumulate) return cudaErrorInvalidValue;
  auto kern = conv_bwd_kernel<PS, VEC, NEED_GY, CH, KMULT, false, PP, HX>;
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
cudaError_t paths_zero_unreached_grad_x(const ConvBwdArgs& a, cudaStream_t stream) {
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
cudaError_t paths_bwd_chunks(const ConvBwdArgs& a, int num_sms, cudaStream_t stream) {
  constexpr int NCH = BwdPlan<PS, paths_bwd_vec<PS>(), NEED_GY>::N;
  cudaError_t err = a.accumulate ? cudaSuccess : paths_zero_unreached_grad_x<PS>(a, stream);
  static_for_host<0, NCH>([&](auto Cc) {
    if (err == cudaSuccess) err = paths_bwd_chunk<PS, NEED_GY, decltype(Cc)::value>(a, num_sms, stream);
  });
  return err;
}

template <int LI, int LS, int LO>
cudaError_t launch_conv_bwd_paths(const ConvBwdArgs& a, int num_sms, cudaStream_t stream) {
  using PS = PathSet<LI, LS, LO>;
  const cudaError_t err = a.grad_edge_vec != nullptr ? paths_bwd_chunks<PS, true>(a, num_sms, stream)
                                                     : paths_bwd_chunks<PS, false>(a, num_sms, stream);
  if (err != cudaSuccess || a.grad_edge_vec == nullptr || a.n_edges == 0) return err;
  const int threads = 256;
  long long nbk = (a.n_edges + threads - 1) / threads;
  if (nbk > (long long)num_sms * 16) nbk = (long long)num_sms * 16;
  const int S = paths_bwd_slices<LI, LS, LO>(a.mult);
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

// The harmonic gradient alone (grad_x and grad_W not wanted): the chunks of
// the plain backward without the T^T g products, then the Jacobian epilogue
// of a.gr_mode.  Partials go to a.grad_sh as in the plain backward.
template <int LI, int LS, int LO>
cudaError_t launch_conv_bwd_gy(const ConvBwdArgs& a, int num_sms, cudaStream_t stream) {
  using PS = PathSet<LI, LS, LO>;
  constexpr int VEC = paths_bwd_vec<PS>();
  constexpr int NCH = BwdPlan<PS, VEC, true>::N;
  if (a.grad_edge_vec == nullptr || a.grad_sh == nullptr) return cudaErrorInvalidValue;
  if (a.n_edges == 0) return cudaSuccess;
  const bool k128 = a.mult == 128 && 128 % (32 * VEC) == 0;
  cudaError_t err = cudaSuccess;
  static_for_host<0, NCH>([&](auto Cc) {
    constexpr int CH = decltype(Cc)::value;
    if (err != cudaSuccess) return;
    err = k128 ? paths_bwd_chunk<PS, true, CH, false, false, 128>(a, num_sms, stream)
               : paths_bwd_chunk<PS, true, CH, false, false, 0>(a, num_sms, stream);
  });
  if (err != cudaSuccess) return err;
  const int threads = 256;
  long long nbk = (a.n_edges + threads - 1) / threads;
  if (nbk > (long long)num_sms * 16) nbk = (long long)num_sms * 16;
  const int S = paths_bwd_slices<LI, LS, LO>(a.mult);
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
template cudaError_t launch_conv_bwd_gy<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(const ConvBwdArgs&, int,
                                                                             cudaStream_t);
template int paths_bwd_slices<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(int);
template cudaError_t launch_conv_paths<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(const ConvFwdArgs&, int,
                                                                           cudaStream_t);
template void conv_path_order<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(int*, int*);
template cudaError_t launch_conv_bwd_paths<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(const ConvBwdArgs&, int,
                                                                                cudaStream_t);

}  // namespace cgtp
