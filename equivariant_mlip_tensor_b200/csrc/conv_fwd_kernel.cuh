// CGTP convolution forward, node-centric over CSR rows, for sm_100a: the one
// kernel template every forward variant of the library is built from.
//
//   out[i][l3,m3][u] = sum_{e in row i} sum_p W_e[p][u] sum_m1 T_e^p[m1][m3] x[j_e][l1,m1][u]
//   T_e^p[m1][m3]    = sum_m2 C^p[m1,m2,m3] Y_e[l2,m2]
//
// ("LunaTP: Enabling Efficient and Scalable Tensor Product for Equivariant
// MLIPs", abstract: node-centric execution, path-group parallelism and reuse;
// the kernel below is our own design for the B200.)
//
// Mapping.  A group of G lanes (G a power of two <= 32) owns one
// (row, channel slice) work item; each lane owns 4 consecutive channels.
// (Optionally one launch per chunk of same-l3 paths.)  The lanes walk the
// row's edges in batches of BT: first every lane computes the harmonics and
// the group's packed T matrices of one edge of the batch (channel
// independent; coefficients are constant-memory operands) into shared
// memory; then the lanes sweep the batch with a two-stage pipeline: while
// edge k is computed, each lane's cp.async copies of edge k+1's weight rows
// (the HBM stream, read once) and of its source's feature rows (L2 resident)
// land in shared memory.  The output rows accumulate in registers and are
// written once; there are no atomics.  Loops over paths and over the
// structural nonzeros of T are unrolled at compile time, so every register
// index is static.
//
// Variants (compile-time):
//  - WSH: one weight row per edge shared by every path (path stride 0;
//    "Tensor Decomposition Networks ...", reply to reviewer oXft) instead of
//    one row per path;
//  - GR::PERPATH: one block of 2 l3 + 1 output rows per path (the per-path
//    messages of the fully connected convolution) instead of summing the
//    paths of one l3;
//  - DD: the double backward's d grad_out in one pass,
//      out = conv(gg_x, W, Y) + conv(x, gg_W, Y) + conv(x, W, Y'),
//    Y' = (dY/dr) gg_r the harmonics' derivative along the edge-vector
//    cotangent: each edge stages W, gg_W, x and gg_x rows and builds both
//    T (from Y) and T' (from Y'), so W and gg_W are read once.
//
// Include after CGTP_DEFINE_CONSTANT_TABLES, conv_common.cuh, vec2.cuh and
// sh.cuh.
#pragma once

namespace cgtp {
namespace {

// Whether the grid is persistent (one wave that loops over the work items)
// or one block per item, and the shared-memory budget per warp (floats) that
// sizes the edge batch.  Blocks of one warp (or of the few warps that split
// one item, kFwdMaxWarps at most) over one item each let the block scheduler
// balance rows of unequal degree: an SM takes a new row as soon as any of
// its blocks finishes one.
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
// Warps that split one item (rows of the forward's graphs with few rows): 1,
// 2 or 4.  More than one measured slower for the forward at the 1 000-atom
// periodic cell (four-warp blocks of its large per-warp staging leave fewer
// warps per SM), so the default keeps one.
#ifndef CGTP_FWD_MAX_WARPS
#define CGTP_FWD_MAX_WARPS 1
#endif
// (the kernels' launch bound follows it: 32 threads by default)
constexpr int kFwdMaxWarps = CGTP_FWD_MAX_WARPS;
#if CGTP_FWD_MINB > 0
#define CGTP_FWD_BOUNDS(KM) __launch_bounds__(kmult_whole_warp(KM, kFwdVec) ? 32 : 32 * kFwdMaxWarps, CGTP_FWD_MINB)
#else
#define CGTP_FWD_BOUNDS(KM) __launch_bounds__(kmult_whole_warp(KM, kFwdVec) ? 32 : 32 * kFwdMaxWarps)
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
// Weight rows in a ring of one slot per staged row (1): the copy of the next
// edge's row of path K is issued once path K of this edge has read its row,
// so the weight rows take one slot each instead of two pipeline stages (the
// gathered feature rows keep two stages); or both in two whole-edge stages (0).
// Smaller edge batches when that lets one wave hold the whole grid (1), not
// below CGTP_FWD_FIT_MIN_BATCH edges.
#ifndef CGTP_FWD_FIT_WAVE
#define CGTP_FWD_FIT_WAVE 1
#endif
#ifndef CGTP_FWD_FIT_MIN_BATCH
#define CGTP_FWD_FIT_MIN_BATCH 4
#endif
#ifndef CGTP_FWD_WRING
#define CGTP_FWD_WRING 1
#endif
constexpr bool kFwdRing = CGTP_FWD_WRING != 0;
// The ring is measured faster for the launches that sum paths into l3 blocks
// (molecules forward 0.2214 -> 0.2126 ms) and slower for the ones that keep
// every path's rows apart (fully connected stage 1, 0.524 -> 0.563 ms): the
// latter keep two whole-edge stages.
template <class GR>
constexpr bool fwd_ring() {
  return kFwdRing && !GR::PERPATH;
}


// One launch over all paths while their unrolled code per edge and lane stays
// within CGTP_FWD_SINGLE_MAX instructions; otherwise one launch per chunk of
// paths with one l3, each within CGTP_FWD_BUDGET (the instruction cache).
#ifndef CGTP_FWD_SINGLE_MAX
#define CGTP_FWD_SINGLE_MAX 1600
#endif
#ifndef CGTP_FWD_BUDGET
#define CGTP_FWD_BUDGET 1100
#endif

// Shared memory of one group of lanes (floats), the same functions on both
// sides of the launch: BT edges of T matrices, the staged rows (ring: one
// slot per weight row and two stages of feature rows; else two stages of
// both), and BT source indices rounded up to a float4.
__host__ __device__ constexpr int fwd_w_floats(int nw, int G) { return nw * G * kFwdVec; }
__host__ __device__ constexpr int fwd_x_floats(int nrow, int G) { return (kStageX ? nrow : 0) * G * kFwdVec; }
__host__ __device__ constexpr int fwd_staging_floats(int w_floats, int x_floats, bool ring) {
  return ring ? w_floats + 2 * x_floats : 2 * (w_floats + x_floats);
}
__host__ __device__ constexpr int fwd_group_floats(int BT, int nt, int w_floats, int x_floats, bool ring) {
  return BT * nt + fwd_staging_floats(w_floats, x_floats, ring) + ((BT + 3) & ~3);
}

// One edge: acc[rows of path K][c] += W[p][c] sum_m1 T[p][m1][m3] x[l1,m1][c]
// for the group's paths.  The edge's weight rows (wst) and source feature
// rows (xst) are this lane's staged copies; with the weight ring each path
// waits for its row's copy group (all but the NWG newest) and, done with the
// row, calls refill(K) for the next edge's copy.
template <class PS, class GR, bool WSH, class Refill>
__device__ __forceinline__ void fwd_edge(const float* __restrict__ T, const float* __restrict__ wst,
                                         const float* __restrict__ xst, int rowf, const float* __restrict__ xg,
                                         int mult, float (&acc)[GR::NOWN][kFwdVec], Refill&& refill) {
  constexpr int NWG = WSH ? 1 : GR::NP;  // weight copy groups per edge
  if constexpr (fwd_ring<GR>()) cp_async_wait<NWG>();  // the feature rows and the first weight row
  float xr[GR::NROW][kFwdVec];
#pragma unroll
  for (int r = 0; r < GR::NROW; ++r) {
    if constexpr (kStageX) VecIO<kFwdVec>::lds(xr[r], xst + r * rowf);
    else VecIO<kFwdVec>::ld(xr[r], xg + r * mult);
  }
  float wsh[kFwdVec];
  if constexpr (WSH) VecIO<kFwdVec>::lds(wsh, wst);  // the one weight row, shared by every path
  static_for<0, GR::NP>([&](auto Kc) {
    constexpr int K = decltype(Kc)::value;
    constexpr int P = GR::D.path[K];
    constexpr int l1 = PS::D.l1[P], l3 = PS::D.l3[P];
    constexpr int tc = PS::D.tcount[P], tb = GR::D.lt[K];
    float wv[kFwdVec];
    if constexpr (WSH) {
#pragma unroll
      for (int c = 0; c < kFwdVec; ++c) wv[c] = wsh[c];
    } else {
      if constexpr (fwd_ring<GR>() && K > 0) cp_async_wait<NWG>();
      VecIO<kFwdVec>::lds(wv, wst + K * rowf);
    }
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
    if constexpr (fwd_ring<GR>()) {  // the path's weight row is read: its slot takes the next edge's
      if constexpr (!WSH) refill(Kc);
      else if constexpr (K == GR::NP - 1) refill(std::integral_constant<int, 0>{});
    }
  });
}

// One edge of the double backward's fused forward, per path:
//   out[m3] += W (sum_m1 T gg_x[m1] + T' x[m1]) + gg_W sum_m1 T x[m1]
// (T' has T's structural pattern: the same path with Y' in place of Y).
// Staged weight rows (wst): W rows (NP), then gg_W rows (NP); xst: x rows,
// then gg_x rows (NROW each).  The ring's waits and refills as in fwd_edge,
// one copy group (W and gg_W rows) per path.
template <class PS, class GR, class Refill>
__device__ __forceinline__ void fwd_edge_dd(const float* __restrict__ T, const float* __restrict__ Td,
                                            const float* __restrict__ wst, const float* __restrict__ xst, int rowf,
                                            float (&acc)[GR::NOWN][kFwdVec], Refill&& refill) {
  constexpr int NP = GR::NP, NR = GR::NROW;
  if constexpr (fwd_ring<GR>()) cp_async_wait<NP>();
  float xr[NR][kFwdVec], gxr[NR][kFwdVec];
#pragma unroll
  for (int r = 0; r < NR; ++r) {
    VecIO<kFwdVec>::lds(xr[r], xst + r * rowf);
    VecIO<kFwdVec>::lds(gxr[r], xst + (NR + r) * rowf);
  }
  static_for<0, NP>([&](auto Kc) {
    constexpr int K = decltype(Kc)::value;
    constexpr int P = GR::D.path[K];
    constexpr int l1 = PS::D.l1[P], l3 = PS::D.l3[P];
    constexpr int tc = PS::D.tcount[P], tb = GR::D.lt[K];
    if constexpr (fwd_ring<GR>() && K > 0) cp_async_wait<NP>();
    float wv[kFwdVec], gwv[kFwdVec];
    VecIO<kFwdVec>::lds(wv, wst + K * rowf);
    VecIO<kFwdVec>::lds(gwv, wst + (NP + K) * rowf);
    constexpr int o3 = l3 * l3 - GR::OWN0;
    if constexpr (2 * l3 + 1 <= 2 * l1 + 1) {
      // tw[m3] = sum T gg_x + T' x (multiplied by W), tg[m3] = sum T x (by gg_W)
      float tw[2 * l3 + 1][kFwdVec], tg[2 * l3 + 1][kFwdVec];
#pragma unroll
      for (int m3 = 0; m3 < 2 * l3 + 1; ++m3)
#pragma unroll
        for (int c = 0; c < kFwdVec; ++c) tw[m3][c] = tg[m3][c] = 0.f;
      static_for<0, (tc + 3) / 4>([&](auto Qc) {
        constexpr int q = decltype(Qc)::value;
        const float4 v4 = *reinterpret_cast<const float4*>(T + tb + 4 * q);
        const float4 d4 = *reinterpret_cast<const float4*>(Td + tb + 4 * q);
        const float tv4[4] = {v4.x, v4.y, v4.z, v4.w}, td4[4] = {d4.x, d4.y, d4.z, d4.w};
        static_for<0, 4>([&](auto Rc) {
          constexpr int k = 4 * q + decltype(Rc)::value;
          if constexpr (k < tc) {
            constexpr int m1 = PS::t_entry_m1(P, k), m3 = PS::t_entry_m3(P, k);
            constexpr int rx = l1 * l1 + l1 + m1 - GR::D.rlo;
            axpy<kFwdVec>(tw[m3 + l3], tv4[decltype(Rc)::value], gxr[rx]);
            axpy<kFwdVec>(tw[m3 + l3], td4[decltype(Rc)::value], xr[rx]);
            axpy<kFwdVec>(tg[m3 + l3], tv4[decltype(Rc)::value], xr[rx]);
          }
        });
      });
#pragma unroll
      for (int m3 = 0; m3 < 2 * l3 + 1; ++m3) {
        vfma<kFwdVec>(acc[o3 + m3], wv, tw[m3]);
        vfma<kFwdVec>(acc[o3 + m3], gwv, tg[m3]);
      }
    } else {
      // qa[m1] = W gg_x + gg_W x (through T), qb[m1] = W x (through T')
      float qa[2 * l1 + 1][kFwdVec], qb[2 * l1 + 1][kFwdVec];
#pragma unroll
      for (int m1 = 0; m1 < 2 * l1 + 1; ++m1) {
        vmul<kFwdVec>(qa[m1], wv, gxr[l1 * l1 + m1 - GR::D.rlo]);
        vfma<kFwdVec>(qa[m1], gwv, xr[l1 * l1 + m1 - GR::D.rlo]);
        vmul<kFwdVec>(qb[m1], wv, xr[l1 * l1 + m1 - GR::D.rlo]);
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
            axpy<kFwdVec>(acc[o3 + m3 + l3], tv4[decltype(Rc)::value], qa[m1 + l1]);
            axpy<kFwdVec>(acc[o3 + m3 + l3], td4[decltype(Rc)::value], qb[m1 + l1]);
          }
        });
      });
    }
    if constexpr (fwd_ring<GR>()) refill(Kc);
  });
}

// GR: the launch's paths (all of them, or one chunk of one l3 block).  A
// chunk that continues an l3 block another chunk of the call started adds
// onto that chunk's rows (GR::FIRST false).
template <class PS, class GR, int KMULT, bool WSH, bool DD>
__global__ void CGTP_FWD_BOUNDS(KMULT)
conv_fwd_kernel(ConvFwdArgs a, int lg_G_rt, int S_rt, int BT, int lg_Q_rt, int lg_W_rt) {
  // KMULT > 0: the multiplicity is a compile-time constant (128: one item of
  // 32 lanes x 4 channels per warp; 64: two items of 16 lanes, whose rows
  // may still be split), so every row offset below folds into an immediate.
  const int mult = KMULT ? KMULT : a.mult;
  constexpr bool WHOLE = kmult_whole_warp(KMULT, kFwdVec);  // one item fills the warp
  const int lg_G = KMULT ? kmult_lg_G(KMULT, kFwdVec) : lg_G_rt;
  const int S = KMULT ? kmult_S(KMULT, kFwdVec) : S_rt;
  const int lg_W = WHOLE ? 0 : lg_W_rt;  // warps of the block that share its items
  constexpr int NI = PS::NI, NO = PS::NO, NS = PS::NS, NT = GR::NT;
  constexpr int NW = (WSH ? 1 : GR::NP) * (DD ? 2 : 1);  // staged weight rows (W, then gg_W)
  constexpr int NXR = GR::NROW * (DD ? 2 : 1);            // staged feature rows (x, then gg_x)
  constexpr int NTE = NT * (DD ? 2 : 1);                  // T floats per edge (T, then T')
  static_assert(!DD || kStageX, "the fused double-backward pass stages its feature rows");
  extern __shared__ float4 smem_f4[];
  float* smem = reinterpret_cast<float*>(smem_f4);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int G = 1 << lg_G, gpw = 32 >> lg_G;
  const int grp = lane >> lg_G, gl = lane & (G - 1);
  constexpr int NWG = WSH ? 1 : GR::NP;                   // weight copy groups per edge
  constexpr bool RING = fwd_ring<GR>();
  const int rowf = G * kFwdVec;                    // floats per staged row
  const int w_floats = fwd_w_floats(NW, G), x_floats = fwd_x_floats(NXR, G);
  const int group_floats = fwd_group_floats(BT, NTE, w_floats, x_floats, RING);
  float* Tg = smem + (warp * gpw + grp) * group_floats;  // warp: this warp within the block
  // staged rows: ring, [NW weight slots][2 stages of NXR feature rows]; else
  // 2 stages of [NW weight rows][NXR feature rows]
  float* St = Tg + BT * NTE;
  auto w_base = [&](int s) { return RING ? St : St + s * (w_floats + x_floats); };
  auto x_base = [&](int s) { return RING ? St + w_floats + s * x_floats : St + s * (w_floats + x_floats) + w_floats; };
  int* Jg = reinterpret_cast<int*>(St + fwd_staging_floats(w_floats, x_floats, RING));

  // The next launch of this call may start on SMs this grid leaves idle
  // (chunks write disjoint rows unless one continues another, and that one
  // waits below).
  grid_dependents_launch();
  if (a.abort_flag != nullptr && (*a.abort_flag & kGraphUnsafeBits)) {  // checked mode, invalid graph
    grid_dependency_wait();
    return;
  }
  // Row split: Q = 2^lg_Q groups of lanes of each of the block's 2^lg_W
  // warps share one work item, part p = warp Q + (group mod Q) taking the
  // row's edges p, p + Q 2^lg_W, ...; their accumulators are summed by
  // shuffles, then across the warps through shared memory (more warps for
  // graphs with few rows).  The block's warps all take the same items.
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
    const int node = active ? int(item / S) : 0;
    const int slice = active ? int(item % S) : 0;
    const int c0 = (slice * G + gl) * kFwdVec;
    int e0 = 0, cnt = 0;  // this group's edges: e0 + part + QT t, t < cnt
    if (active) {
      e0 = __ldg(a.row_ptr + node);
      const int deg = __ldg(a.row_ptr + node + 1) - e0;
      cnt = deg > part ? (deg - part + QT - 1) >> lg_QT : 0;
      e0 += part;
    }
    const int maxdeg = __reduce_max_sync(0xffffffffu, cnt);
    float acc[GR::NOWN][kFwdVec];
#pragma unroll
    for (int r = 0; r < GR::NOWN; ++r)
#pragma unroll
      for (int c = 0; c < kFwdVec; ++c) acc[r][c] = 0.f;

    // copies of edge slot k of the current batch (this lane's channels only):
    // w_src gives the edge's weight rows (this lane's channels; negative when
    // the slot holds no edge of this group), issue_w copies those of copy
    // group J into the weight rows at wdst, issue_x the feature rows into xdst
    auto w_src = [&](int b0, int k) -> long long {
      if (!(active && b0 + k < cnt)) return -1;
      return (long long)(e0 + ((b0 + k) << lg_QT)) * (WSH ? 1 : PS::NP) * mult + c0;
    };
    auto issue_w = [&](long long src, auto Jc, float* wdst) {
      constexpr int J = decltype(Jc)::value;
      if (src < 0) return;
      float* dst = wdst + gl * kFwdVec;
      if constexpr (WSH) {
        cp_async_w<kFwdVec>(dst, a.w + src, wpol);
      } else {
        constexpr int P = GR::D.path[J];
        cp_async_w<kFwdVec>(dst + J * rowf, a.w + src + P * mult, wpol);
        if constexpr (DD) cp_async_w<kFwdVec>(dst + (GR::NP + J) * rowf, a.w2 + src + P * mult, wpol);
      }
    };
    auto issue_x = [&](int b0, int k, float* xdst) {
      if constexpr (kStageX || DD) {
        if (!(active && b0 + k < cnt)) return;
        float* dst = xdst + gl * kFwdVec;
        constexpr int rlo = GR::D.rlo;
        const float* xrow = a.x + ((long long)Jg[k] * NI + rlo) * mult + c0;
#pragma unroll
        for (int r = 0; r < GR::NROW; ++r) VecIO<kFwdVec>::cp_async(dst + r * rowf, xrow + r * mult);
        if constexpr (DD) {
          const float* x2row = a.x2 + ((long long)Jg[k] * NI + rlo) * mult + c0;
#pragma unroll
          for (int r = 0; r < GR::NROW; ++r) VecIO<kFwdVec>::cp_async(dst + (GR::NROW + r) * rowf, x2row + r * mult);
        }
      }
    };

    for (int b0 = 0; b0 < maxdeg; b0 += BT) {
      // sources of every slot, then the first slot's copies, so that they fly
      // while the T matrices of the batch are computed
      for (int k = gl; k < BT; k += G) {
        if (active && b0 + k < cnt) {
          const int e = e0 + ((b0 + k) << lg_QT);
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
      // Copy groups.  Ring: X(k) (the feature rows of edge k) is committed at
      // the start of edge k - 1 and W(k, J) (copy group J of its weight rows)
      // during edge k - 1 once path J is done, so exactly NWG groups follow
      // W(k, J) when path J of edge k reads it (W(k, J+1..), X(k+1),
      // W(k+1, ..J-1)), and more follow X(k): every wait leaves the NWG
      // newest.  The batch's first edge is copied in the same order.  Without
      // the ring, one group per edge and a wait for all but the newest.
      {
        const long long src0 = w_src(b0, 0);
        if constexpr (RING) {
          issue_x(b0, 0, x_base(0));
          cp_async_commit();
          static_for<0, NWG>([&](auto Jc) {
            issue_w(src0, Jc, w_base(0));
            cp_async_commit();
          });
        } else {
          static_for<0, NWG>([&](auto Jc) { issue_w(src0, Jc, w_base(0)); });
          issue_x(b0, 0, x_base(0));
          cp_async_commit();
        }
      }
      for (int k = gl; k < BT; k += G) {
        if (active && b0 + k < cnt) {
          const int e = e0 + ((b0 + k) << lg_QT);
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
            edge_sh<PS::LS>(a.sh, a.edge_vec, e, Y);
            compute_T_grp<PS, GR>(Y, Tg + k * NT);
          }
        }
      }
      __syncwarp();
      for (int k = 0; k < nb; ++k) {
        const long long src_next = k + 1 < nb ? w_src(b0, k + 1) : -1;
        if (k + 1 < nb) {
          if constexpr (!RING) static_for<0, NWG>([&](auto Jc) { issue_w(src_next, Jc, w_base((k + 1) & 1)); });
          issue_x(b0, k + 1, x_base((k + 1) & 1));
        }
        cp_async_commit();
        if constexpr (!RING) cp_async_wait<1>();  // this lane's copies of edge k have landed
        // ring: the slot of copy group J takes edge k + 1's rows (an empty
        // group past the batch keeps the count)
        auto refill = [&](auto Jc) {
          issue_w(src_next, Jc, w_base(0));
          cp_async_commit();
        };
        if (active && b0 + k < cnt) {
          constexpr int rlo = GR::D.rlo;
          const float* wst = w_base(k & 1) + gl * kFwdVec;
          const float* xst = x_base(k & 1) + gl * kFwdVec;
          if constexpr (DD)
            fwd_edge_dd<PS, GR>(Tg + k * NT, Tg + (BT + k) * NT, wst, xst, rowf, acc, refill);
          else
            fwd_edge<PS, GR, WSH>(Tg + k * NT, wst, xst, rowf, a.x + ((long long)Jg[k] * NI + rlo) * mult + c0, mult,
                                  acc, refill);
        }
      }
      __syncwarp();
    }
    // the row's parts: sum the groups of one item (lanes gl + G part)
    for (int sh = 1; sh < Q; sh <<= 1) {
#pragma unroll
      for (int r = 0; r < GR::NOWN; ++r)
#pragma unroll
        for (int c = 0; c < kFwdVec; ++c) acc[r][c] += __shfl_xor_sync(0xffffffffu, acc[r][c], sh * G);
    }
    if (lg_W > 0) {
      // then the warps' sums, in warp order, by warp 0: each warp's part-0
      // groups leave theirs at the start of their own shared-memory region
      // (NOWN rows of G x 4 floats, within the group's region)
      cp_async_wait<0>();
      __syncthreads();
      const bool head = (grp & (Q - 1)) == 0;
      if (warp > 0 && head) {
#pragma unroll
        for (int r = 0; r < GR::NOWN; ++r) VecIO<kFwdVec>::st(Tg + r * rowf + gl * kFwdVec, acc[r]);
      }
      __syncthreads();
      if (warp == 0 && head) {
        for (int w = 1; w < nwarps; ++w) {
          const float* theirs = smem + (w * gpw + grp) * group_floats + gl * kFwdVec;
#pragma unroll
          for (int r = 0; r < GR::NOWN; ++r) {
            float v[kFwdVec];
            VecIO<kFwdVec>::lds(v, theirs + r * rowf);
#pragma unroll
            for (int c = 0; c < kFwdVec; ++c) acc[r][c] += v[c];
          }
        }
      }
      __syncthreads();
    }
    if constexpr (GR::PERPATH) {
      // t[node][m3][rank][u] of this l3 block, rank = the path's place among
      // the block's paths
      if (active && part == 0) {
        constexpr int n3 = 2 * GR::KEY + 1;
        static_for<0, GR::NP>([&](auto Kc) {
          constexpr int K = decltype(Kc)::value;
#pragma unroll
          for (int m3 = 0; m3 < n3; ++m3)
            VecIO<kFwdVec>::st(a.out + (((long long)node * n3 + m3) * GR::NPK + GR::PL0 + K) * mult + c0,
                               acc[K * n3 + m3]);
        });
      }
    } else if (active && part == 0) {
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
  // Complete only after the preceding launch: a grid launched with
  // programmatic stream serialization that never waited could otherwise
  // complete before its predecessor, and whatever the stream runs after the
  // last launch of the chain (the next call, or a caller's kernel writing
  // into memory this call has finished with) would then overlap a launch that
  // is still running.  A no-op for a grid launched in plain stream order.
  grid_dependency_wait();
}

template <class PS, class GR, bool WSH, bool DD = false>
cudaError_t launch_fwd_group(const ConvFwdArgs& a, int num_sms, bool pdl, cudaStream_t stream) {
  int G, lg_G, S;
  lane_geometry(a.mult, kFwdVec, G, lg_G, S);
  const int gpw = 32 / G;
  const int mul = DD ? 2 : 1;  // the fused double-backward pass stages and builds everything twice
  const int w_floats = fwd_w_floats((WSH ? 1 : GR::NP) * mul, G), x_floats = fwd_x_floats(GR::NROW * mul, G);
  // compile-time multiplicities: 128 for every launch, 64 for the plain
  // forward (the others keep the run-time one there)
  constexpr bool kAllow64 = CGTP_KMULT64 && !WSH && !DD && !GR::PERPATH;
  auto kern = a.mult == 128               ? conv_fwd_kernel<PS, GR, 128, WSH, DD>
              : (kAllow64 && a.mult == 64) ? conv_fwd_kernel<PS, GR, kAllow64 ? 64 : 0, WSH, DD>
                                           : conv_fwd_kernel<PS, GR, 0, WSH, DD>;
  const long long items = (long long)a.n_nodes * S;
  constexpr bool RING = fwd_ring<GR>();
  int BT = pick_batch_staged(gpw, GR::NT * mul, fwd_staging_floats(w_floats, x_floats, RING), CGTP_FWD_BATCH_FLOATS,
                             CGTP_FWD_MAX_BATCH);
  int lg_W = 0;
  const int lg_Q = row_split(items, gpw, num_sms, a.mult == 128 ? 1 : kFwdMaxWarps, &lg_W);
  // fewer warps per item when the block's shared memory would not fit, or a
  // group's region could not hold the warps' sums (NOWN rows of G x 4 floats)
  const int gfl = fwd_group_floats(BT, GR::NT * mul, w_floats, x_floats, RING);
  while (lg_W > 0 && (sizeof(float) * (size_t)gfl * (gpw << lg_W) > smem_limit() || GR::NOWN * G * kFwdVec > gfl))
    --lg_W;
  const int threads = 32 << lg_W;
  const long long items_per_block = (long long)(gpw >> lg_Q);
  long long blocks = (items + items_per_block - 1) / items_per_block;
  // the kernel's indexing reaches gpw groups x warps of group_floats each
  auto smem_of = [&](int bt) {
    return sizeof(float) * (size_t)fwd_group_floats(bt, GR::NT * mul, w_floats, x_floats, RING) * gpw * (threads / 32);
  };
  if (CGTP_FWD_FIT_WAVE && blocks > 1) {
    // A grid that one wave would hold with smaller edge batches (few rows,
    // e.g. one periodic cell) gets the largest batch that makes it fit: the
    // T matrices are most of a group's shared memory.
    static int regs_of[3] = {-1, -1, -1};  // per kernel of this instantiation (multiplicity 128, 64, run time)
    int& regs = regs_of[a.mult == 128 ? 0 : (kAllow64 && a.mult == 64) ? 1 : 2];
    if (regs < 0) {
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return cudaGetLastError();
      regs = fa.numRegs;
    }
    if (blocks > (long long)num_sms * resident_blocks_per_sm(smem_of(BT), regs, threads)) {
      for (int bt = BT - 1; bt >= CGTP_FWD_FIT_MIN_BATCH; --bt)
        if (blocks <= (long long)num_sms * resident_blocks_per_sm(smem_of(bt), regs, threads)) {
          BT = bt;
          break;
        }
    }
  }
  const size_t smem = smem_of(BT);
  cudaError_t err = check_smem(smem);
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  long long cap = 0x7fffffffLL;  // the kernel loops over items beyond the grid
  if (CGTP_FWD_PERSISTENT) {
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
    if (err != cudaSuccess) return err;
    cap = (long long)num_sms * (per_sm < 1 ? 1 : per_sm);
  }
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return launch_kernel(kern, dim3((unsigned)blocks), dim3(threads), smem, stream, pdl, a, lg_G, S, BT, lg_Q, lg_W);
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
// the fused double-backward forward carries about three times the code per
// path (three T products): its own budget (730 measured best of 366 ... 2000)
#ifndef CGTP_DD_FWD_BUDGET
#define CGTP_DD_FWD_BUDGET 730
#endif
template <class PS>
using FwdPlanDD = Plan<PS, kByL3, kFwdVec, false, CGTP_DD_FWD_BUDGET>;

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

// The forward over every path (summed by l3 blocks): one launch when all
// paths fit one unrolled edge body, else one launch per chunk of same-l3
// paths, every chunk after the first overlapping its predecessor.
template <class PS, bool WSH>
cudaError_t launch_fwd_all(const ConvFwdArgs& a, int num_sms, cudaStream_t stream) {
  if constexpr (fwd_all_cost<PS>() <= CGTP_FWD_SINGLE_MAX) {
    // all paths in one launch (it writes every output row, reached or not)
    return launch_fwd_group<PS, Grp<PS, kAll, 0>, WSH>(a, num_sms, false, stream);
  } else {
    cudaError_t err = a.accumulate ? cudaSuccess : zero_unreached_out<PS>(a, stream);
    static_for_host<0, FwdPlan<PS>::N>([&](auto Cc) {
      constexpr int CH = decltype(Cc)::value;
      if (err == cudaSuccess)
        err = launch_fwd_group<PS, ChunkGrp<PS, FwdPlan<PS>, CH, kByL3>, WSH>(a, num_sms, CH > 0, stream);
    });
    return err;
  }
}

// The double backward's d grad_out in one pass per chunk of same-l3 paths
// (a.x2 = gg_x, a.w2 = gg_W, a.gr_dir = gg_r); overwrites a.out.
template <class PS>
cudaError_t launch_fwd_dd(const ConvFwdArgs& a, int num_sms, cudaStream_t stream) {
  if (a.x2 == nullptr || a.w2 == nullptr || a.gr_dir == nullptr || a.accumulate || a.sh != nullptr)
    return cudaErrorInvalidValue;
  if constexpr (3 * fwd_all_cost<PS>() <= CGTP_FWD_SINGLE_MAX) {
    return launch_fwd_group<PS, Grp<PS, kAll, 0>, false, true>(a, num_sms, false, stream);
  } else {
    cudaError_t err = zero_unreached_out<PS>(a, stream);
    static_for_host<0, FwdPlanDD<PS>::N>([&](auto Cc) {
      constexpr int CH = decltype(Cc)::value;
      if (err == cudaSuccess)
        err = launch_fwd_group<PS, ChunkGrp<PS, FwdPlanDD<PS>, CH, kByL3>, false, true>(a, num_sms, CH > 0,
                                                                                         stream);
    });
    return err;
  }
}

}  // namespace
}  // namespace cgtp
