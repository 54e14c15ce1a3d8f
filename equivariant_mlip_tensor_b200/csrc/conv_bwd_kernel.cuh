// CGTP convolution backward, node-centric over sources (CSC), for sm_100a:
// the one kernel template every backward variant of the library is built
// from.
//
// For edge e = (j -> i) with T_e^p[m1][m3] = sum_m2 C^p[m1,m2,m3] Y_e[l2,m2]:
//   h_p[m1][u]      = sum_m3 T_e^p[m1][m3] g[i][l3,m3][u]
//   grad_x[j][l1,m1][u] += W_e[p][u] h_p[m1][u]
//   grad_W[e][p][u] = sum_m1 x[j][l1,m1][u] h_p[m1][u]
//   grad_Y[e][l2,m2] = sum_p sum_{m1,m3} C^p[m1,m2,m3] sum_u W_e[p][u] x[j][l1,m1][u] g[i][l3,m3][u]
// (the adjoints of the bilinear convolution; cf. the closed-form gradients
// of a bilinear tensor product in "Tensor Decomposition Networks ...",
// reply to reviewer S6y1, and the derivative computation of "LunaTP ...",
// abstract).
//
// A group of G lanes owns one (source node j, channel slice); it keeps x[j]
// and the grad_x[j] accumulator in registers for the whole CSC row, so W is
// read once, grad_W is written once and grad_x needs no atomics.  grad_Y is
// reduced over the group's channels through shared memory and written, per
// channel slice, to a workspace [slices][E][NS]; sh_backward then sums the
// slices and applies the harmonic Jacobian to give grad_edge_vec.
//
// Variants (compile-time flags VAR):
//  - kVarExt: per-edge harmonics given by the caller and results added onto
//    the outputs (the double backward's first-order passes);
//  - kVarPerPath: grad_out holds one gradient block per path (the per-path
//    message layout of the fully connected convolution);
//  - kVarWShared: one weight row per edge shared by every path; grad_w[e] is
//    the sum over paths (chunks then run in plain stream order, each adding
//    onto the row the previous chunks wrote);
//  - kVarDD: the double backward's d x, d W and edge-vector terms in one pass
//    (see bwd_edge_dd): W and gg_W staged per edge, x and gg_x held per
//    source, T from Y and T' from Y' = (dY/dr) gg_r.
//
// Include after CGTP_DEFINE_CONSTANT_TABLES, conv_common.cuh, vec2.cuh and
// sh.cuh.
#pragma once

namespace cgtp {

enum : int { kVarExt = 1, kVarPerPath = 2, kVarWShared = 8, kVarDD = 16 };

namespace {

// Persistent grid or one block per item, and the shared-memory budget per
// warp (floats) that sizes the edge batch (as in the forward: blocks of one
// warp, or of the few warps that split one item, let the block scheduler
// balance the rows).
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
// (blocks of the compile-time multiplicity keep one warp, and their launch
// bound says so: with a bound of 128 threads the molecules backward took
// 0.518 ms instead of 0.504)
constexpr int kBwdMaxWarps = 4;
// Warps that split one item (source rows of graphs with few rows): 1, 2 or 4.
#ifndef CGTP_BWD_MAX_WARPS
#define CGTP_BWD_MAX_WARPS 4
#endif
#if CGTP_BWD_MINB > 0
#define CGTP_BWD_BOUNDS(KM) __launch_bounds__(kmult_whole_warp(KM, kBwdVec) ? 32 : 32 * kBwdMaxWarps, CGTP_BWD_MINB)
#else
#define CGTP_BWD_BOUNDS(KM) __launch_bounds__(kmult_whole_warp(KM, kBwdVec) ? 32 : 32 * kBwdMaxWarps)
#endif
// Channels per lane (float4: measured faster than 2 at every shape with
// one-warp blocks and budgeted chunks).
#ifndef CGTP_BWD_VEC
#define CGTP_BWD_VEC 4
#endif
constexpr int kBwdVec = CGTP_BWD_VEC;
// The per-path-layout variant (fully connected convolution) with the
// compile-time multiplicity 128 too (1: its backward at molecules 1.97 ->
// 1.76 ms, bit-identical), or only the run-time one (0).
#ifndef CGTP_PP_KMULT
#define CGTP_PP_KMULT 1
#endif
// The harmonic Jacobian epilogue launched with programmatic dependent launch
// (1) or in plain stream order (0), and the largest l1 block's chain of
// chunks on the caller's stream, the others on side lanes (1), or the
// smallest block's (0).  Together: molecules backward 0.509 -> 0.503 ms
// (0.355 -> 0.351 ms without the Jacobian), bit-identical.
#ifndef CGTP_SH_PDL
#define CGTP_SH_PDL 1
#endif
#ifndef CGTP_BWD_LONG_MAIN
#define CGTP_BWD_LONG_MAIN 1
#endif
// Programmatic dependent launch between the chunks of one backward call
// (1) or plain stream order (0).
#ifndef CGTP_BWD_PDL
#define CGTP_BWD_PDL 1
#endif

// Unrolled instructions per edge and lane allowed in one backward launch
// (measured at the molecules shape: 1100 -> 1400 took the backward from
// 0.535 to 0.507 ms; 1700 and more lose again, and a launch near 3000
// instructions doubles the time on instruction fetch), and in one launch of
// the fused double-backward pass (two T products per path: 730 measured
// best of 488 ... 2000).
#ifndef CGTP_BWD_BUDGET
#define CGTP_BWD_BUDGET 1400
#endif
#ifndef CGTP_BWD_BUDGET_L3
#define CGTP_BWD_BUDGET_L3 800  // l = 3 chunks carry more registers per path
#endif
#ifndef CGTP_DD_BWD_BUDGET
#define CGTP_DD_BWD_BUDGET 730
#endif
template <class PS>
constexpr int bwd_budget() {
  return PS::LI >= 3 || PS::LO >= 3 ? CGTP_BWD_BUDGET_L3 : CGTP_BWD_BUDGET;
}
template <class PS>
constexpr int dd_bwd_budget() {  // l = 3: scaled like the plain backward's
  return PS::LI >= 3 || PS::LO >= 3 ? CGTP_DD_BWD_BUDGET * CGTP_BWD_BUDGET_L3 / 1100 : CGTP_DD_BWD_BUDGET;
}

// The fused double-backward pass carries a little over twice the code per
// path (two T products, two harmonic-gradient sums): its own budget.
// Merge small l1 blocks into the next one's launch when the whole blocks fit
// the budget (1), or one launch per block at least (0).
#ifndef CGTP_BWD_MERGE
#define CGTP_BWD_MERGE 1
#endif
// The fused double-backward pass plans its chunks as if the harmonic
// gradient were always wanted, so that d x and d W come out of the same
// chunks (and bit for bit the same) whichever outputs a call requests.
// With CGTP_BWD_MERGE_TAIL a merged run of whole blocks also takes the paths
// that would form the next block's last (small) chunk when they fit, and that
// block's other chunks continue its rows: one launch and one fixed per-edge
// cost fewer (the fused double-backward pass at the molecules shape: 6 -> 5
// chunks, 1.68 -> 1.65 ms; the plain backward's plans there are unchanged).
#ifndef CGTP_BWD_MERGE_TAIL
#define CGTP_BWD_MERGE_TAIL 1
#endif
template <class PS, bool NEED_GY, int VAR = 0>
using BwdPlan = Plan<PS, kByL1, kBwdVec, ((VAR & kVarDD) != 0) || NEED_GY,
                     (VAR & kVarDD) ? dd_bwd_budget<PS>() : bwd_budget<PS>(), (1 << 30), CGTP_BWD_MERGE != 0,
                     CGTP_BWD_MERGE != 0 && CGTP_BWD_MERGE_TAIL != 0>;

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

// Staged rows per edge: weight rows (one per path, or the one shared row)
// and output-gradient rows (the chunk's l3 range, or every path's own block).
template <class PS, class GR, int VAR>
constexpr int bwd_staged_rows() {
  return ((VAR & kVarWShared) ? 1 : GR::NP) * ((VAR & kVarDD) ? 2 : 1) +
         ((VAR & kVarPerPath) ? pp_rowoff<PS, GR>(GR::NP) : GR::NROW);
}

// Shared memory (floats), the same functions on both sides of the launch:
// per group of lanes BT edges of T matrices, two pipeline stages and two
// index arrays of BT ints rounded up to a float4; after all groups, one
// grad_Y reduction buffer of NS rows of G + 4 floats per group.
__host__ __device__ constexpr int bwd_group_floats(int BT, int nt, int stage_floats) {
  return BT * nt + 2 * stage_floats + 2 * ((BT + 3) & ~3);
}
__host__ __device__ constexpr int bwd_red_floats(int ns, int G) { return ns * (G + 4); }

// One edge of the CSC row, the paths of one group (l1 = GR's value).  Per
// path, with h[m1] = sum_m3 T[m1][m3] g[m3] (one pass over the structural
// nonzeros of T):
//   grad_x[m1] += W h[m1],   grad_W = sum_m1 x[m1] h[m1],
// and, for grad_Y, the channel sums sum_u W x[m1] g[m3] of every T entry
// contracted with the CG coefficients.  Paths are visited in (l2, ...) order
// so that only one l2 block of the grad_Y partial is live at a time; each
// finished block goes to this lane's column of the shared reduction buffer
// (gyrow, row stride rs).  The edge's weight rows and its destination's
// output-gradient rows come from this lane's pipeline stage.
template <class PS, class GR, int VEC, bool NEED_GY, int VAR>
__device__ __forceinline__ void bwd_edge(const float* __restrict__ T, const float* __restrict__ stage, int rowf,
                                         const float (&xr)[GR::NOWN][VEC], float* __restrict__ gwrow, bool acc, int mult,
                                         float (&gx)[GR::NOWN][VEC], float* __restrict__ gyrow, int rs) {
  constexpr bool PP = (VAR & kVarPerPath) != 0, WSH = (VAR & kVarWShared) != 0;
  constexpr int NW = WSH ? 1 : GR::NP;  // staged weight rows
  float gy[PS::NS];
  float gws[VEC];  // WSH: grad of the shared weight row, summed over this chunk's paths
#pragma unroll
  for (int c = 0; c < VEC; ++c) gws[c] = 0.f;
  static_for<0, GR::NP>([&](auto Kc) {
    constexpr int K = decltype(Kc)::value;
    constexpr int P = GR::D.path[K];
    constexpr int l1 = PS::D.l1[P], l3 = PS::D.l3[P];
    [[maybe_unused]] constexpr int l2 = PS::D.l2[P];
    constexpr int tb = GR::D.lt[K], tc = PS::D.tcount[P];
    constexpr int o1 = l1 * l1 - GR::OWN0;  // the path's x / grad_x rows among the chunk's own
    // staged row of grad_out[l3, m3 = -l3] (of this path's own rows when PP)
    constexpr int g0 = NW + (PP ? pp_rowoff<PS, GR>(K) : l3 * l3 - GR::D.rlo);
    if constexpr (NEED_GY && GR::D.first_l2[K]) {
#pragma unroll
      for (int m2 = 0; m2 < 2 * l2 + 1; ++m2) gy[l2 * l2 + m2] = 0.f;
    }
    float wv[VEC];
    VecIO<VEC>::lds(wv, stage + (WSH ? 0 : K) * rowf);
    float gv[2 * l3 + 1][VEC], h[2 * l1 + 1][VEC];
#pragma unroll
    for (int m3 = 0; m3 < 2 * l3 + 1; ++m3) VecIO<VEC>::lds(gv[m3], stage + (g0 + m3) * rowf);
#pragma unroll
    for (int m1 = 0; m1 < 2 * l1 + 1; ++m1)
#pragma unroll
      for (int c = 0; c < VEC; ++c) h[m1][c] = 0.f;
    [[maybe_unused]] float xw[2 * l1 + 1][VEC];  // W x, for the grad_Y channel sums
    if constexpr (NEED_GY) {
#pragma unroll
      for (int m1 = 0; m1 < 2 * l1 + 1; ++m1) vmul<VEC>(xw[m1], wv, xr[o1 + m1]);
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
    {
      if constexpr (WSH) {
#pragma unroll
        for (int m1 = 0; m1 < 2 * l1 + 1; ++m1) {
          vfma<VEC>(gx[o1 + m1], wv, h[m1]);
          vfma<VEC>(gws, xr[o1 + m1], h[m1]);
        }
      } else {
        float gw[VEC];
#pragma unroll
        for (int c = 0; c < VEC; ++c) gw[c] = 0.f;
#pragma unroll
        for (int m1 = 0; m1 < 2 * l1 + 1; ++m1) {
          vfma<VEC>(gx[o1 + m1], wv, h[m1]);
          vfma<VEC>(gw, xr[o1 + m1], h[m1]);
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
    }
    if constexpr (NEED_GY && GR::D.last_l2[K]) {
#pragma unroll
      for (int m2 = 0; m2 < 2 * l2 + 1; ++m2) gyrow[(l2 * l2 + m2) * rs] = gy[l2 * l2 + m2];
    }
  });
  if constexpr (WSH) {
    if (gwrow != nullptr) {
      if (acc) {  // an earlier chunk of this call wrote the row: add onto it
        float prev[VEC];
        VecIO<VEC>::ld(prev, gwrow);
#pragma unroll
        for (int c = 0; c < VEC; ++c) gws[c] += prev[c];
      }
      VecIO<VEC>::st_stream(gwrow, gws);
    }
  }
}

// One edge of the double backward's fused pass, per path, with
// h[m1] = sum_m3 T[m1][m3] g[m3] and h'[m1] = sum_m3 T'[m1][m3] g[m3]:
//   d_x[m1]  += gg_W h[m1] + W h'[m1]
//   d_W       = sum_m1 gg_x[m1] h[m1] + x[m1] h'[m1]
//   A[l2,m2] += C sum_u (W gg_x[m1] + gg_W x[m1]) g[m3]   (contracted with dY/dr)
//   B[l2,m2] += C sum_u W x[m1] g[m3]                      (with d2Y/dr2 gg_r)
// (the derivatives of <gg_x, grad_x> + <gg_W, grad_W> + <gg_r, grad_r>).
// Stage layout: W rows (NP), gg_W rows (NP), grad_out rows (NROW).
template <class PS, class GR, int VEC, bool NEED_GY>
__device__ __forceinline__ void bwd_edge_dd(const float* __restrict__ T, const float* __restrict__ Td,
                                            const float* __restrict__ stage, int rowf,
                                            const float (&xr)[GR::NOWN][VEC], const float (&gxr)[GR::NOWN][VEC],
                                            float* __restrict__ gwrow, int mult, float (&gx)[GR::NOWN][VEC],
                                            float* __restrict__ gyrowA, float* __restrict__ gyrowB, int rs) {
  constexpr int NP = GR::NP;
  float gyA[PS::NS], gyB[PS::NS];
  static_for<0, NP>([&](auto Kc) {
    constexpr int K = decltype(Kc)::value;
    constexpr int P = GR::D.path[K];
    constexpr int l1 = PS::D.l1[P], l3 = PS::D.l3[P];
    [[maybe_unused]] constexpr int l2 = PS::D.l2[P];
    constexpr int tb = GR::D.lt[K], tc = PS::D.tcount[P];
    constexpr int g0 = 2 * NP + l3 * l3 - GR::D.rlo;  // staged row of grad_out[l3, m3 = -l3]
    constexpr int o1 = l1 * l1 - GR::OWN0;             // the path's rows among the chunk's own
    if constexpr (NEED_GY && GR::D.first_l2[K]) {
#pragma unroll
      for (int m2 = 0; m2 < 2 * l2 + 1; ++m2) gyA[l2 * l2 + m2] = gyB[l2 * l2 + m2] = 0.f;
    }
    float wv[VEC], gwv[VEC];
    VecIO<VEC>::lds(wv, stage + K * rowf);
    VecIO<VEC>::lds(gwv, stage + (NP + K) * rowf);
    float gv[2 * l3 + 1][VEC], h[2 * l1 + 1][VEC], hd[2 * l1 + 1][VEC];
#pragma unroll
    for (int m3 = 0; m3 < 2 * l3 + 1; ++m3) VecIO<VEC>::lds(gv[m3], stage + (g0 + m3) * rowf);
#pragma unroll
    for (int m1 = 0; m1 < 2 * l1 + 1; ++m1)
#pragma unroll
      for (int c = 0; c < VEC; ++c) h[m1][c] = hd[m1][c] = 0.f;
    [[maybe_unused]] float pa[2 * l1 + 1][VEC], pb[2 * l1 + 1][VEC];
    if constexpr (NEED_GY) {
#pragma unroll
      for (int m1 = 0; m1 < 2 * l1 + 1; ++m1) {
        vmul<VEC>(pa[m1], wv, gxr[o1 + m1]);
        vfma<VEC>(pa[m1], gwv, xr[o1 + m1]);
        vmul<VEC>(pb[m1], wv, xr[o1 + m1]);
      }
    }
    static_for<0, (tc + 3) / 4>([&](auto Qc) {
      constexpr int q = decltype(Qc)::value;
      const float4 v4 = *reinterpret_cast<const float4*>(T + tb + 4 * q);
      const float4 d4 = *reinterpret_cast<const float4*>(Td + tb + 4 * q);
      const float tv4[4] = {v4.x, v4.y, v4.z, v4.w}, td4[4] = {d4.x, d4.y, d4.z, d4.w};
      static_for<0, 4>([&](auto Rc) {
        constexpr int k = 4 * q + decltype(Rc)::value;
        if constexpr (k < tc) {
          constexpr int m1 = PS::t_entry_m1(P, k), m3 = PS::t_entry_m3(P, k);
          axpy<VEC>(h[m1 + l1], tv4[decltype(Rc)::value], gv[m3 + l3]);
          axpy<VEC>(hd[m1 + l1], td4[decltype(Rc)::value], gv[m3 + l3]);
          if constexpr (NEED_GY) {
            const float aa = vdot<VEC>(pa[m1 + l1], gv[m3 + l3]);
            const float ab = vdot<VEC>(pb[m1 + l1], gv[m3 + l3]);
            static_for<0, 2 * l2 + 1>([&](auto M2c) {
              constexpr int m2 = decltype(M2c)::value - l2;
              if constexpr (cg_allowed(l1, l2, l3, m1, m2, m3)) {
                constexpr int ti = table_index(l1, l2, l3, m1, m2, m3);
                gyA[l2 * l2 + l2 + m2] = fmaf(c_cg[ti], aa, gyA[l2 * l2 + l2 + m2]);
                gyB[l2 * l2 + l2 + m2] = fmaf(c_cg[ti], ab, gyB[l2 * l2 + l2 + m2]);
              }
            });
          }
        }
      });
    });
    float gw[VEC];
#pragma unroll
    for (int c = 0; c < VEC; ++c) gw[c] = 0.f;
#pragma unroll
    for (int m1 = 0; m1 < 2 * l1 + 1; ++m1) {
      vfma<VEC>(gx[o1 + m1], gwv, h[m1]);
      vfma<VEC>(gx[o1 + m1], wv, hd[m1]);
      vfma<VEC>(gw, gxr[o1 + m1], h[m1]);
      vfma<VEC>(gw, xr[o1 + m1], hd[m1]);
    }
    if (gwrow != nullptr) VecIO<VEC>::st_stream(gwrow + P * mult, gw);
    if constexpr (NEED_GY && GR::D.last_l2[K]) {
#pragma unroll
      for (int m2 = 0; m2 < 2 * l2 + 1; ++m2) {
        gyrowA[(l2 * l2 + m2) * rs] = gyA[l2 * l2 + m2];
        gyrowB[(l2 * l2 + m2) * rs] = gyB[l2 * l2 + m2];
      }
    }
  });
}

// One launch per chunk (paths of one l1 block): grad_x rows of that block
// (written by the block's first chunk, accumulated by the others), grad_W
// of the chunk's paths and a partial grad_Y over them.
template <class PS, bool NEED_GY, int CH, int KMULT, int VAR>
__global__ void CGTP_BWD_BOUNDS(KMULT)
conv_bwd_kernel(ConvBwdArgs a, int lg_G_rt, int S_rt, int BT, int slice_base_rt, int lg_Q_rt, int lg_W_rt) {
  constexpr int VEC = kBwdVec;
  constexpr bool EXT = (VAR & kVarExt) != 0, PP = (VAR & kVarPerPath) != 0;
  constexpr bool WSH = (VAR & kVarWShared) != 0, DD = (VAR & kVarDD) != 0;
  static_assert(!DD || (VAR == kVarDD), "the fused double-backward pass is a variant of its own");
  // KMULT > 0: the multiplicity is a compile-time constant (128: one item of
  // 32 lanes x VEC channels per warp; 64: two items of 16 lanes, whose rows
  // may still be split), so every row offset below folds into an immediate.
  const int mult = KMULT ? KMULT : a.mult;
  constexpr bool WHOLE = kmult_whole_warp(KMULT, VEC);  // one item fills the warp
  const int lg_G = KMULT ? kmult_lg_G(KMULT, VEC) : lg_G_rt;
  const int S = KMULT ? kmult_S(KMULT, VEC) : S_rt;
  const int slice_base = KMULT ? CH * S : slice_base_rt;
  const int lg_W = WHOLE ? 0 : lg_W_rt;  // warps of the block that share its items
  using PL = BwdPlan<PS, NEED_GY, VAR & kVarDD>;
  using GR = ChunkGrp<PS, PL, CH, kByL1>;
  constexpr int OWN0 = GR::OWN0;  // first x / grad_x row of the chunk's l1 blocks
  constexpr int NI = PS::NI, NO = PS::NO, NS = PS::NS, NR = GR::NOWN, NT = GR::NT;
  constexpr int NW = (WSH ? 1 : GR::NP) * (DD ? 2 : 1);     // staged weight rows (W, then gg_W)
  constexpr int NTE = NT * (DD ? 2 : 1);                   // T floats per edge (T, then T')
  constexpr int NROWS = bwd_staged_rows<PS, GR, VAR>();
  constexpr unsigned GY_MASK = touched_sh_mask<PS, GR>();  // harmonics this chunk's paths reach
  extern __shared__ float4 smem_f4[];
  float* smem = reinterpret_cast<float*>(smem_f4);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int G = 1 << lg_G, gpw = 32 >> lg_G;
  const int grp = lane >> lg_G, gl = lane & (G - 1);
  const int rowf = G * VEC;
  const int stage_floats = NROWS * rowf;
  const int group_floats = bwd_group_floats(BT, NTE, stage_floats);
  float* Tg = smem + (warp * gpw + grp) * group_floats;
  float* St = Tg + BT * NTE;
  int* Eg = reinterpret_cast<int*>(St + 2 * stage_floats);
  int* Ig = Eg + ((BT + 3) & ~3);
  // grad_Y reduction buffer, per group of lanes: NS rows (one per harmonic)
  // of G lane partials, row stride rs = G + 4 (float4 aligned, and rows read
  // by the 8 lanes of one 128-bit access phase fall in distinct banks)
  const int rs = G + 4;
  // (two such buffers in the fused double-backward pass: its A and B sums)
  float* red = smem + (gpw << lg_W) * group_floats +
               (warp * gpw + grp) * bwd_red_floats(NS, G) * (DD ? 2 : 1);
  [[maybe_unused]] const int slices_total = S * PL::N;  // the B partials follow the A partials

  // The next chunk of this call may start on SMs this grid leaves idle: no
  // chunk reads what another writes, except a chunk that adds onto an
  // earlier chunk's grad_x rows, and that one waits for it below.
  grid_dependents_launch();
  if (a.abort_flag != nullptr && (*a.abort_flag & kGraphUnsafeBits)) {  // checked mode, invalid graph
    grid_dependency_wait();
    return;
  }
  // Row split: Q = 2^lg_Q groups of lanes of each of the block's 2^lg_W
  // warps share one work item (source row), part p = warp Q + (group mod Q)
  // taking the row's edges p, p + Q 2^lg_W, ...; their grad_x accumulators
  // are summed by shuffles, then across the warps through shared memory.
  // The block's warps all take the same items.
  // (a compile-time multiplicity fills the warp with one item: no split
  // inside the warp)
  // (nor across warps: one warp per item)
  const int lg_Q = WHOLE ? 0 : lg_Q_rt;
  const int lg_QT = lg_Q + lg_W, nwarps = 1 << lg_W;
  const int Q = 1 << lg_Q, QT = 1 << lg_QT, part = (warp << lg_Q) | (grp & (Q - 1));
  const int ipw = gpw >> lg_Q;  // items per block
  const uint64_t wpol = stream_policy();
  const long long n_items = (long long)a.n_nodes * S;
  for (long long base = (long long)blockIdx.x * ipw; base < n_items; base += (long long)gridDim.x * ipw) {
    const long long item = base + (grp >> lg_Q);
    const bool active = item < n_items;
    const long long node = active ? item / S : 0;
    const int slice = active ? int(item % S) : 0;
    const int c0 = (slice * G + gl) * VEC;
    int k0 = 0, cnt = 0;  // this group's CSC slots: k0 + part + QT t, t < cnt
    if (active) {
      k0 = __ldg(a.csc_ptr + node);
      const int deg = __ldg(a.csc_ptr + node + 1) - k0;
      cnt = deg > part ? (deg - part + QT - 1) >> lg_QT : 0;
      k0 += part;
    }
    const int maxdeg = __reduce_max_sync(0xffffffffu, cnt);
    float xr[NR][VEC], gx[NR][VEC];
    [[maybe_unused]] float gxr[NR][VEC];  // DD: gg_x of the source
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      if (active) {
        VecIO<VEC>::ld(xr[r], a.x + (node * NI + OWN0 + r) * mult + c0);
        if constexpr (DD) VecIO<VEC>::ld(gxr[r], a.x2 + (node * NI + OWN0 + r) * mult + c0);
      } else {
#pragma unroll
        for (int c = 0; c < VEC; ++c) {
          xr[r][c] = 0.f;
          if constexpr (DD) gxr[r][c] = 0.f;
        }
      }
#pragma unroll
      for (int c = 0; c < VEC; ++c) gx[r][c] = 0.f;
    }

    // copies of edge slot k of the current batch into stage s (this lane's channels only)
    auto issue = [&](int b0, int k, int s) {
      if (!(active && b0 + k < cnt)) return;
      float* dst = St + s * stage_floats + gl * VEC;
      if constexpr (WSH) {
        cp_async_w<VEC>(dst, a.w + (long long)Eg[k] * mult + c0, wpol);
      } else {
        const float* wrow = a.w + (long long)Eg[k] * PS::NP * mult + c0;
        [[maybe_unused]] const float* w2row = DD ? a.w2 + (long long)Eg[k] * PS::NP * mult + c0 : nullptr;
        static_for<0, GR::NP>([&](auto Kc) {
          constexpr int K = decltype(Kc)::value;
          constexpr int P = GR::D.path[K];
          cp_async_w<VEC>(dst + K * rowf, wrow + P * mult, wpol);
          if constexpr (DD) cp_async_w<VEC>(dst + (GR::NP + K) * rowf, w2row + P * mult, wpol);
        });
      }
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
            VecIO<VEC>::cp_async(dst + (NW + ro + m3) * rowf, base + (long long)m3 * npk * mult);
        });
      } else {
        constexpr int rlo = GR::D.rlo;
        const float* grow = a.grad_out + ((long long)Ig[k] * NO + rlo) * mult + c0;
#pragma unroll
        for (int r = 0; r < GR::NROW; ++r) VecIO<VEC>::cp_async(dst + (NW + r) * rowf, grow + r * mult);
      }
    };

    for (int b0 = 0; b0 < maxdeg; b0 += BT) {
      for (int k = gl; k < BT; k += G) {
        const int kk = k0 + ((b0 + k) << lg_QT);
        if (active && b0 + k < cnt) {
          const int e = __ldg(a.csc_edge + kk);
          float Y[NS];
          if constexpr (DD) {
            // Y and Y' = (dY/dr) gg_r in one evaluation
            Dual1 yd[NS];
            sh_dir_of_vec<PS::LS>(__ldg(a.edge_vec + 3 * e), __ldg(a.edge_vec + 3 * e + 1),
                                  __ldg(a.edge_vec + 3 * e + 2), __ldg(a.gr_dir + 3 * e),
                                  __ldg(a.gr_dir + 3 * e + 1), __ldg(a.gr_dir + 3 * e + 2), yd);
            float Yd[NS];
#pragma unroll
            for (int b = 0; b < NS; ++b) {
              Y[b] = yd[b].v;
              Yd[b] = yd[b].e;
            }
            compute_T_grp<PS, GR>(Y, Tg + k * NT);
            compute_T_grp<PS, GR>(Yd, Tg + (BT + k) * NT);
          } else {
            edge_sh<PS::LS>(EXT ? a.sh : nullptr, a.edge_vec, e, Y);
            compute_T_grp<PS, GR>(Y, Tg + k * NT);
          }
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
        const bool valid = active && b0 + k < cnt;
        int e = 0;
        if (valid) {
          e = Eg[k];
          float* gwrow = nullptr;
          if (a.grad_w != nullptr) gwrow = a.grad_w + (long long)e * (WSH ? 1 : PS::NP) * mult + c0;
          if constexpr (DD) {
            bwd_edge_dd<PS, GR, VEC, NEED_GY>(Tg + k * NT, Tg + (BT + k) * NT,
                                               St + (k & 1) * stage_floats + gl * VEC, rowf, xr, gxr, gwrow,
                                               mult, gx, red + gl, red + NS * rs + gl, rs);
          } else {
            // WSH: every chunk after the first adds onto the row (plain stream order)
            const bool acc = (WSH && CH > 0) || (EXT && a.accumulate != 0);
            bwd_edge<PS, GR, VEC, NEED_GY, VAR>(Tg + k * NT, St + (k & 1) * stage_floats + gl * VEC, rowf, xr,
                                                 gwrow, acc, mult, gx, red + gl, rs);
          }
        }
        if constexpr (NEED_GY) {
          __syncwarp();
          if (valid) {
            // column sums; harmonics the chunk never reaches get 0
            auto column_sums = [&](const float* rbuf, float* dst) {
              for (int b = gl; b < NS; b += G) {
                float v = 0.f;
                if ((GY_MASK >> b) & 1u) {
                  const float* row = rbuf + b * rs;
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
            };
            column_sums(red, a.grad_sh + ((long long)(slice_base + slice) * a.n_edges + e) * NS);
            if constexpr (DD)
              column_sums(red + NS * rs,
                          a.grad_sh + ((long long)(slices_total + slice_base + slice) * a.n_edges + e) * NS);
          }
          __syncwarp();
        }
      }
      __syncwarp();
    }
    // the row's parts: sum the groups of one item (lanes gl + G part)
    for (int sh = 1; sh < Q; sh <<= 1) {
#pragma unroll
      for (int r = 0; r < NR; ++r)
#pragma unroll
        for (int c = 0; c < VEC; ++c) gx[r][c] += __shfl_xor_sync(0xffffffffu, gx[r][c], sh * G);
    }
    if (lg_W > 0) {
      // then the warps' sums, in warp order, by warp 0: each warp's part-0
      // groups leave theirs at the start of their own shared-memory region
      // (NR rows of G x VEC floats, within the group's region)
      cp_async_wait<0>();
      __syncthreads();
      const bool head = (grp & (Q - 1)) == 0;
      if (warp > 0 && head) {
#pragma unroll
        for (int r = 0; r < NR; ++r) VecIO<VEC>::st(Tg + r * rowf + gl * VEC, gx[r]);
      }
      __syncthreads();
      if (warp == 0 && head) {
        for (int w = 1; w < nwarps; ++w) {
          const float* theirs = smem + (w * gpw + grp) * group_floats + gl * VEC;
#pragma unroll
          for (int r = 0; r < NR; ++r) {
            float v[VEC];
            VecIO<VEC>::lds(v, theirs + r * rowf);
#pragma unroll
            for (int c = 0; c < VEC; ++c) gx[r][c] += v[c];
          }
        }
      }
      __syncthreads();
    }
    if (active && part == 0 && a.grad_x != nullptr) {
      if (!GR::FIRST || (EXT && a.accumulate)) {
        // rows of an l1 block that an earlier chunk of this call wrote (wait
        // for that grid, the preceding launch), or the caller's values
        if constexpr (!GR::FIRST) grid_dependency_wait();
#pragma unroll
        for (int r = 0; r < NR; ++r) {
          float prev[VEC];
          VecIO<VEC>::ld(prev, a.grad_x + (node * NI + OWN0 + r) * mult + c0);
#pragma unroll
          for (int c = 0; c < VEC; ++c) gx[r][c] += prev[c];
        }
      }
#pragma unroll
      for (int r = 0; r < NR; ++r) VecIO<VEC>::st(a.grad_x + (node * NI + OWN0 + r) * mult + c0, gx[r]);
    }
  }
  // Complete only after the preceding launch: a grid launched with
  // programmatic stream serialization that never waited (no grad_x rows to
  // add onto, or no grad_x at all) could otherwise complete before its
  // predecessor, and what the stream runs after the chain would overlap a
  // launch that is still running.  A no-op in plain stream order.
  grid_dependency_wait();
}

// grad_edge_vec[e] (= or +=) (dY_e/dr_e)^T sum_s grad_sh[s][e].  Launched
// with programmatic dependent launch after the chunks: the Jacobian needs only
// the edge vectors, so it is evaluated before waiting for the chunks' partials.
template <int LS>
__global__ void sh_backward_kernel(int n_edges, int S, const float* __restrict__ edge_vec,
                                   const float* __restrict__ grad_sh, float* __restrict__ grad_edge_vec, int add) {
  constexpr int NS = (LS + 1) * (LS + 1);
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n_edges;
       e += (long long)gridDim.x * blockDim.x) {
    Dual3 Y[NS];
    sh_grad_of_vec<LS>(edge_vec[3 * e], edge_vec[3 * e + 1], edge_vec[3 * e + 2], Y);
    grid_dependency_wait();  // the partials (and the caller's grad_edge_vec) from here on
    float g[NS];
#pragma unroll
    for (int b = 0; b < NS; ++b) g[b] = 0.f;
    for (int s = 0; s < S; ++s) {
      const float* src = grad_sh + ((long long)s * n_edges + e) * NS;
#pragma unroll
      for (int b = 0; b < NS; ++b) g[b] += src[b];
    }
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
  grid_dependency_wait();  // complete only after the chunks (threads without an edge too)
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

// channel lanes per group (G) and channel slices (S) of the backward
inline void bwd_geometry(int mult, int& G, int& lg_G, int& S) { lane_geometry(mult, kBwdVec, G, lg_G, S); }

// One partial grad_Y per (chunk, channel slice) (the fused double-backward
// pass writes two such sets).
template <class PS, int VAR = 0>
int bwd_slices(int mult) {
  int G, lg_G, S;
  bwd_geometry(mult, G, lg_G, S);
  return S * BwdPlan<PS, true, VAR & kVarDD>::N;
}

// Launch chunk CH of variant VAR (the double backward's harmonics input or
// accumulate mode selects the kExt kernel at run time).
template <class PS, bool NEED_GY, int CH, int VAR>
cudaError_t launch_bwd_chunk(const ConvBwdArgs& a, int num_sms, cudaStream_t stream, bool pdl) {
  using GR = ChunkGrp<PS, BwdPlan<PS, NEED_GY, VAR & kVarDD>, CH, kByL1>;
  constexpr int mul = (VAR & kVarDD) ? 2 : 1;  // T and T', two reduction buffers
  int G, lg_G, S;
  bwd_geometry(a.mult, G, lg_G, S);
  const int gpw = 32 / G;
  const int stage_floats = bwd_staged_rows<PS, GR, VAR>() * G * kBwdVec;
  const int BT = pick_batch(gpw, GR::NT * mul, stage_floats, CGTP_BWD_BATCH_FLOATS, CGTP_BWD_MAX_BATCH);
  // the kernel's indexing reaches gpw groups x warps of group_floats, then
  // (with NEED_GY) as many reduction buffers
  const long long items = (long long)a.n_nodes * S;
  const bool ext = a.sh != nullptr || a.accumulate;
  // the compile-time multiplicity for the common case (one warp per item),
  // and 64 for the plain backward
  constexpr bool kAllow128 = CGTP_PP_KMULT || (VAR & kVarPerPath) == 0;
  constexpr bool kAllow64 = CGTP_KMULT64 && (VAR & (kVarPerPath | kVarWShared | kVarDD)) == 0;
  const bool kmult = !ext && kAllow128 && a.mult == 128;
  const bool kmult64 = !ext && kAllow64 && a.mult == 64;
  int lg_W = 0;
  const int lg_Q = row_split(items, gpw, num_sms, kmult ? 1 : CGTP_BWD_MAX_WARPS, &lg_W);
  const int gfl = bwd_group_floats(BT, GR::NT * mul, stage_floats);
  const int per_group = gfl + (NEED_GY ? bwd_red_floats(PS::NS, G) * mul : 0);
  // fewer warps per item when the block's shared memory would not fit, or a
  // group's region could not hold the warps' sums (NOWN rows of G x VEC floats)
  while (lg_W > 0 && (sizeof(float) * (size_t)per_group * (gpw << lg_W) > smem_limit() || GR::NOWN * G * kBwdVec > gfl))
    --lg_W;
  const int threads = 32 << lg_W;
  const size_t groups = (size_t)gpw << lg_W;
  const size_t smem = sizeof(float) * (groups * gfl + (NEED_GY ? groups * bwd_red_floats(PS::NS, G) * mul : 0));
  cudaError_t err = check_smem(smem);
  if (err != cudaSuccess) return err;
  const long long items_per_block = (long long)(gpw >> lg_Q);
  const long long blocks = (items + items_per_block - 1) / items_per_block;
  if (ext && (VAR & (kVarPerPath | kVarWShared | kVarDD))) return cudaErrorInvalidValue;  // not built
  constexpr int kExtVar = (VAR & (kVarPerPath | kVarWShared | kVarDD)) ? VAR : (VAR | kVarExt);
  auto kern = ext ? conv_bwd_kernel<PS, NEED_GY, CH, 0, kExtVar>
              : kmult   ? conv_bwd_kernel<PS, NEED_GY, CH, kAllow128 ? 128 : 0, VAR>
              : kmult64 ? conv_bwd_kernel<PS, NEED_GY, CH, kAllow64 ? 64 : 0, VAR>
                        : conv_bwd_kernel<PS, NEED_GY, CH, 0, VAR>;
  err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  long long cap = 0x7fffffffLL;  // the kernel loops over items beyond the grid
  if (CGTP_BWD_PERSISTENT) {
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
    if (err != cudaSuccess) return err;
    cap = (long long)num_sms * (per_sm < 1 ? 1 : per_sm);
  }
  long long nb = blocks > cap ? cap : blocks;
  if (nb < 1) nb = 1;
  return launch_kernel(kern, dim3((unsigned)nb), dim3(threads), smem, stream, CGTP_BWD_PDL && pdl, a, lg_G,
                       S, BT, CH * S, lg_Q, lg_W);
}

// grad_x blocks that no path reaches (l1 with no path) are zero.
template <class PS>
cudaError_t zero_unreached_grad_x(const ConvBwdArgs& a, cudaStream_t stream) {
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

// Every chunk of variant VAR.  LANES: chunks of different l1 blocks write
// disjoint outputs (their own grad_x rows, their own paths' grad_W rows,
// their own grad_Y partial slices), so each l1 block's chunks run on a lane
// of their own, forked from the caller's stream and joined back before the
// call's next launch: the latency-bound small blocks then fill the SMs beside
// the large ones.  Within a lane (and without lanes), a chunk that continues
// an l1 block overlaps its predecessor through programmatic dependent launch
// and waits for it before adding to its rows.  Shared-weight chunks all add
// onto one gradient row per edge, so they run in plain stream order.
template <class PS, bool NEED_GY, int VAR, bool LANES>
cudaError_t launch_bwd_chunks(const ConvBwdArgs& a, int num_sms, cudaStream_t stream) {
  using PL = BwdPlan<PS, NEED_GY, VAR & kVarDD>;
  constexpr int NCH = PL::N;
  constexpr int NCHAINS = PL::CHAINS;  // chunks that continue rows follow their predecessor on its lane
  constexpr bool kPdl = (VAR & kVarWShared) == 0;
  cudaError_t err = a.accumulate ? cudaSuccess : zero_unreached_grad_x<PS>(a, stream);
  if (err != cudaSuccess) return err;
  if constexpr (!LANES || NCHAINS <= 1 || !kPdl) {
    static_for_host<0, NCH>([&](auto Cc) {
      constexpr int CH = decltype(Cc)::value;
      if (err == cudaSuccess) err = launch_bwd_chunk<PS, NEED_GY, CH, VAR>(a, num_sms, stream, kPdl && CH > 0);
    });
    return err;
  } else {
    std::lock_guard<std::mutex> turn(side_lanes_mutex(kLanesBwd));
    SideLanes* L = nullptr;
    err = side_lanes(kLanesBwd, &L);
    if (err == cudaSuccess) err = lanes_fork(L, NCHAINS - 1, stream);
    static_for_host<0, NCH>([&](auto Cc) {
      constexpr int CH = decltype(Cc)::value;
      // the chain's lane; lane 0 is the caller's stream (with
      // CGTP_BWD_LONG_MAIN the last chain, the largest l1 block's, takes it:
      // the epilogue then follows the longest chain in stream order)
      constexpr int lane = CGTP_BWD_LONG_MAIN ? NCHAINS - 1 - PL::P.chain[CH] : PL::P.chain[CH];
      if (err == cudaSuccess)
        err = launch_bwd_chunk<PS, NEED_GY, CH, VAR>(a, num_sms, lane == 0 ? stream : L->side[lane - 1],
                                                     !PL::P.first_of_key[CH]);
    });
    if (L != nullptr) {  // join even after an error, so no lane is left forked
      const cudaError_t e = lanes_join(L, NCHAINS - 1, stream);
      if (err == cudaSuccess) err = e;
    }
    return err;
  }
}

// The harmonic Jacobian epilogue: grad_edge_vec from the summed partials
// (gr_mode 0/1), or the double backward's Hessian-vector term (gr_mode 2/3).
template <int LS>
cudaError_t launch_sh_backward(const ConvBwdArgs& a, int slices, int num_sms, cudaStream_t stream) {
  const int threads = 256;
  long long nbk = (a.n_edges + threads - 1) / threads;
  if (nbk > (long long)num_sms * 16) nbk = (long long)num_sms * 16;
  if (a.gr_mode >= 2) {
    if (a.gr_dir == nullptr) return cudaErrorInvalidValue;
    sh_backward_hess_kernel<LS><<<(unsigned)nbk, threads, 0, stream>>>(a.n_edges, slices, a.edge_vec, a.grad_sh,
                                                                      a.gr_dir, a.grad_edge_vec, a.gr_mode == 2);
  } else {
    return launch_kernel(sh_backward_kernel<LS>, dim3((unsigned)nbk), dim3(threads), 0, stream, CGTP_SH_PDL != 0,
                         (int)a.n_edges, slices, a.edge_vec, (const float*)a.grad_sh, a.grad_edge_vec,
                         (int)(a.gr_mode == 1));
  }
  return cudaGetLastError();
}

// The whole backward of variant VAR: the chunks (with grad_Y partials when
// grad_edge_vec is wanted), then the harmonic Jacobian epilogue.
template <class PS, int VAR, bool LANES>
cudaError_t launch_bwd_all(const ConvBwdArgs& a, int num_sms, cudaStream_t stream) {
  const cudaError_t err = a.grad_edge_vec != nullptr ? launch_bwd_chunks<PS, true, VAR, LANES>(a, num_sms, stream)
                                                     : launch_bwd_chunks<PS, false, VAR, LANES>(a, num_sms, stream);
  if (err != cudaSuccess || a.grad_edge_vec == nullptr || a.n_edges == 0) return err;
  return launch_sh_backward<PS::LS>(a, bwd_slices<PS>(a.mult), num_sms, stream);
}

// The fused double backward's edge-vector term:
//   d_r[e] = (dY/dr)^T A_e + sum_b B_e,b (d2Y_b/dr2) gg_r[e]
// with A and B the two partial sets (each summed over its slices); one
// evaluation gives the Jacobian and the Hessian-vector product.
template <int LS>
__global__ void sh_backward_dd_kernel(int n_edges, int S, const float* __restrict__ edge_vec,
                                      const float* __restrict__ gsh, const float* __restrict__ q,
                                      float* __restrict__ d_r) {
  constexpr int NS = (LS + 1) * (LS + 1);
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n_edges;
       e += (long long)gridDim.x * blockDim.x) {
    float A[NS], B[NS];
#pragma unroll
    for (int b = 0; b < NS; ++b) A[b] = B[b] = 0.f;
    for (int s = 0; s < S; ++s) {
      const float* pa = gsh + ((long long)s * n_edges + e) * NS;
      const float* pb = gsh + ((long long)(S + s) * n_edges + e) * NS;
#pragma unroll
      for (int b = 0; b < NS; ++b) {
        A[b] += pa[b];
        B[b] += pb[b];
      }
    }
    HDual Y[NS];
    sh_hess_of_vec<LS>(edge_vec[3 * e], edge_vec[3 * e + 1], edge_vec[3 * e + 2], q[3 * e], q[3 * e + 1],
                       q[3 * e + 2], Y);
    float d0 = 0.f, d1 = 0.f, d2 = 0.f;
#pragma unroll
    for (int b = 0; b < NS; ++b) {
      d0 = fmaf(A[b], Y[b].d0.v, fmaf(B[b], Y[b].d0.e, d0));
      d1 = fmaf(A[b], Y[b].d1.v, fmaf(B[b], Y[b].d1.e, d1));
      d2 = fmaf(A[b], Y[b].d2.v, fmaf(B[b], Y[b].d2.e, d2));
    }
    d_r[3 * e] = d0;
    d_r[3 * e + 1] = d1;
    d_r[3 * e + 2] = d2;
  }
}

// The fused double backward's source-centric pass: every chunk (the l1
// blocks on forked lanes), then the edge-vector epilogue when
// a.grad_edge_vec is wanted.  a.x2 = gg_x, a.w2 = gg_W, a.gr_dir = gg_r;
// a.grad_x = d_x, a.grad_w = d_W, a.grad_edge_vec = d_r (each nullable);
// a.grad_sh holds 2 x bwd_slices<PS, kVarDD> partial slices.
template <class PS>
cudaError_t launch_bwd_dd(const ConvBwdArgs& a, int num_sms, cudaStream_t stream) {
  if (a.x2 == nullptr || a.w2 == nullptr || a.gr_dir == nullptr || a.sh != nullptr || a.accumulate)
    return cudaErrorInvalidValue;
  if (a.grad_edge_vec != nullptr && a.grad_sh == nullptr) return cudaErrorInvalidValue;
  const cudaError_t err = a.grad_edge_vec != nullptr ? launch_bwd_chunks<PS, true, kVarDD, true>(a, num_sms, stream)
                                                     : launch_bwd_chunks<PS, false, kVarDD, true>(a, num_sms, stream);
  if (err != cudaSuccess || a.grad_edge_vec == nullptr || a.n_edges == 0) return err;
  const int threads = 256;
  long long nbk = (a.n_edges + threads - 1) / threads;
  if (nbk > (long long)num_sms * 16) nbk = (long long)num_sms * 16;
  sh_backward_dd_kernel<PS::LS><<<(unsigned)nbk, threads, 0, stream>>>(
      a.n_edges, bwd_slices<PS, kVarDD>(a.mult), a.edge_vec, a.grad_sh, a.gr_dir, a.grad_edge_vec);
  return cudaGetLastError();
}

}  // namespace
}  // namespace cgtp
