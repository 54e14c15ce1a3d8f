// CP-decomposed CG tensor product of batched pairs, for sm_100a.
//
//   z[b][:, u] = A (B^T x[b][:, u] (*) C^T y[b][:, u])      ((*) elementwise)
//
// with factor matrices A [d3][R], B [d1][R], C [d2][R] shared by every pair
// and channel, d1 = (L_in+1)^2, d2 = (L_sh+1)^2, d3 = (L_out+1)^2
// ("Tensor Decomposition Networks for Accelerating Machine Learning Force
// Field Computations", reply to reviewer S6y1: the forward map and the
// closed-form backward g_x = (g_z^T A (*) C^T y) B^T, g_y = (g_z^T A (*) B^T x) C^T).
// The factor gradients follow from the same trilinear form, summed over pairs
// and channels: g_A = sum g_z (s (*) t)^T, g_B = sum x (q (*) t)^T,
// g_C = sum y (q (*) s)^T with s = B^T x, t = C^T y, q = A^T g_z.
//
// One thread per (pair, channel); consecutive threads take consecutive
// channels, so every feature load and store is coalesced.  A block copies the
// factors into shared memory transposed to [r][row] (rows padded to a multiple
// of four floats), so that one rank component is a few broadcast float4 loads.
// The rank loop is a runtime loop; the row loops are unrolled at the shape's
// compile-time dimensions.  The factor gradients are reduced without atomics:
// a block of 64 threads walks a fixed run of 64-item tiles; per tile it stages
// the items' rank vectors (s (*) t, q (*) t, q (*) s) and inputs in shared
// memory and adds their contraction over the tile's items into its own
// partial of every factor entry (each thread owns fixed entries); a second
// kernel sums the at most 512 block partials with a fixed reduction tree
// (bit-reproducible).
#include "common.cuh"
#include "launch.h"

namespace cgtp {
namespace {

constexpr int kCpFwdThreads = 128;
constexpr int kCpBwdItems = kCpItemsPerTile;  // items (and threads) per backward block with factor gradients
constexpr int kCpBwdThreads = 128;
constexpr int kCpItemStride = kCpBwdItems + 4;  // staged rows: 16-byte aligned, rows r and r+1 in distinct banks

constexpr int pad4(int d) { return (d + 3) & ~3; }

template <int LI, int LS, int LO>
struct CpShape {
  static constexpr int D1 = (LI + 1) * (LI + 1), D2 = (LS + 1) * (LS + 1), D3 = (LO + 1) * (LO + 1);
  static constexpr int P1 = pad4(D1), P2 = pad4(D2), P3 = pad4(D3);
  static constexpr int PT = P1 + P2 + P3;  // transposed factor floats per rank component
};

// Factors into shared memory as [r][row] with rows padded by zeros (reads in
// the global row-major order, so that a warp reads consecutive floats).
template <int D, int P>
__device__ __forceinline__ void load_factor(const float* __restrict__ F, int R, float* Ft) {
  for (int idx = threadIdx.x; idx < D * R; idx += blockDim.x) Ft[(idx % R) * P + idx / R] = F[idx];
  if constexpr (P > D)
    for (int idx = threadIdx.x; idx < (P - D) * R; idx += blockDim.x) Ft[(idx / (P - D)) * P + D + idx % (P - D)] = 0.f;
}
template <class S>
__device__ __forceinline__ void load_factors(const float* __restrict__ A, const float* __restrict__ B,
                                             const float* __restrict__ C, int R, float* Bt, float* Ct, float* At) {
  load_factor<S::D1, S::P1>(B, R, Bt);
  load_factor<S::D2, S::P2>(C, R, Ct);
  load_factor<S::D3, S::P3>(A, R, At);
}

// sum_i f[i] v[i] over D entries of a padded factor row.
template <int D>
__device__ __forceinline__ float row_dot(const float* __restrict__ f, const float (&v)[D]) {
  float s = 0.f;
#pragma unroll
  for (int i4 = 0; i4 < pad4(D) / 4; ++i4) {
    const float4 q = reinterpret_cast<const float4*>(f)[i4];
    const float fq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int c = 0; c < 4; ++c)
      if (4 * i4 + c < D) s = fmaf(fq[c], v[4 * i4 + c], s);
  }
  return s;
}

// acc[i] += f[i] a over D entries of a padded factor row.
template <int D>
__device__ __forceinline__ void row_axpy(float (&acc)[D], const float* __restrict__ f, float a) {
#pragma unroll
  for (int i4 = 0; i4 < pad4(D) / 4; ++i4) {
    const float4 q = reinterpret_cast<const float4*>(f)[i4];
    const float fq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int c = 0; c < 4; ++c)
      if (4 * i4 + c < D) acc[4 * i4 + c] = fmaf(fq[c], a, acc[4 * i4 + c]);
  }
}

template <int D>
__device__ __forceinline__ void load_rows(float (&v)[D], const float* __restrict__ p, long long b, int u, int mult,
                                          bool ok) {
#pragma unroll
  for (int i = 0; i < D; ++i) v[i] = ok ? __ldg(p + (b * D + i) * mult + u) : 0.f;
}

template <class S>
__global__ void __launch_bounds__(kCpFwdThreads) cp_fwd_kernel(CPArgs a) {
  extern __shared__ float4 cps4[];
  float* Bt = reinterpret_cast<float*>(cps4);
  float* Ct = Bt + a.rank * S::P1;
  float* At = Ct + a.rank * S::P2;
  load_factors<S>(a.A, a.B, a.C, a.rank, Bt, Ct, At);
  __syncthreads();
  const long long item = (long long)blockIdx.x * kCpFwdThreads + threadIdx.x;
  const long long items = (long long)a.batch * a.mult;
  if (item >= items) return;
  const long long b = item / a.mult;
  const int u = (int)(item % a.mult);
  float x[S::D1], y[S::D2], z[S::D3];
  load_rows<S::D1>(x, a.x, b, u, a.mult, true);
  load_rows<S::D2>(y, a.y, b, u, a.mult, true);
#pragma unroll
  for (int k = 0; k < S::D3; ++k) z[k] = 0.f;
  for (int r = 0; r < a.rank; ++r) {
    const float p = row_dot<S::D1>(Bt + r * S::P1, x) * row_dot<S::D2>(Ct + r * S::P2, y);
    row_axpy<S::D3>(z, At + r * S::P3, p);
  }
#pragma unroll
  for (int k = 0; k < S::D3; ++k) a.z[(b * S::D3 + k) * a.mult + u] = z[k];
}

// Backward of one item (pair, channel), and, with GF, the staging of its rank
// vectors and inputs for the factor gradients (column t of the tile buffers).
template <class S, bool GF>
__device__ __forceinline__ void cp_bwd_item(const CPArgs& a, long long item, int t, const float* Bt, const float* Ct,
                                            const float* At, float* Pst, float* Pqt, float* Pqs, float* Xs,
                                            float* Ys, float* Gs) {
  const long long items = (long long)a.batch * a.mult;
  const bool ok = item < items;
  const long long b = ok ? item / a.mult : 0;
  const int u = ok ? (int)(item % a.mult) : 0;
  float x[S::D1], y[S::D2], g[S::D3], gx[S::D1], gy[S::D2];
  load_rows<S::D1>(x, a.x, b, u, a.mult, ok);
  load_rows<S::D2>(y, a.y, b, u, a.mult, ok);
  load_rows<S::D3>(g, a.grad_z, b, u, a.mult, ok);
#pragma unroll
  for (int i = 0; i < S::D1; ++i) gx[i] = 0.f;
#pragma unroll
  for (int j = 0; j < S::D2; ++j) gy[j] = 0.f;
  for (int r = 0; r < a.rank; ++r) {
    const float s = row_dot<S::D1>(Bt + r * S::P1, x);
    const float tt = row_dot<S::D2>(Ct + r * S::P2, y);
    const float q = row_dot<S::D3>(At + r * S::P3, g);
    const float qt = q * tt, qs = q * s;
    row_axpy<S::D1>(gx, Bt + r * S::P1, qt);
    row_axpy<S::D2>(gy, Ct + r * S::P2, qs);
    if constexpr (GF) {
      Pst[r * kCpItemStride + t] = s * tt;
      Pqt[r * kCpItemStride + t] = qt;
      Pqs[r * kCpItemStride + t] = qs;
    }
  }
  if (ok) {
    if (a.grad_x != nullptr) {
#pragma unroll
      for (int i = 0; i < S::D1; ++i) a.grad_x[(b * S::D1 + i) * a.mult + u] = gx[i];
    }
    if (a.grad_y != nullptr) {
#pragma unroll
      for (int j = 0; j < S::D2; ++j) a.grad_y[(b * S::D2 + j) * a.mult + u] = gy[j];
    }
  }
  if constexpr (GF) {
#pragma unroll
    for (int i = 0; i < S::D1; ++i) Xs[i * kCpItemStride + t] = x[i];
#pragma unroll
    for (int j = 0; j < S::D2; ++j) Ys[j * kCpItemStride + t] = y[j];
#pragma unroll
    for (int k = 0; k < S::D3; ++k) Gs[k * kCpItemStride + t] = g[k];
  }
}

// Input gradients only: one thread per item.
template <class S>
__global__ void __launch_bounds__(kCpBwdThreads) cp_bwd_kernel(CPArgs a) {
  extern __shared__ float4 cps4[];
  float* Bt = reinterpret_cast<float*>(cps4);
  float* Ct = Bt + a.rank * S::P1;
  float* At = Ct + a.rank * S::P2;
  load_factors<S>(a.A, a.B, a.C, a.rank, Bt, Ct, At);
  __syncthreads();
  const long long item = (long long)blockIdx.x * kCpBwdThreads + threadIdx.x;
  if (item >= (long long)a.batch * a.mult) return;
  cp_bwd_item<S, false>(a, item, threadIdx.x, Bt, Ct, At, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr);
}

// Input gradients and the block's partial of every factor-gradient entry,
// [g_A (D3 x R) | g_B (D1 x R) | g_C (D2 x R)], over the block's run of tiles.
template <class S>
__global__ void __launch_bounds__(kCpBwdItems) cp_bwd_factors_kernel(CPArgs a, long long tiles, long long tpb) {
  constexpr int T = kCpBwdItems;
  extern __shared__ float4 cps4[];
  const int R = a.rank;
  const int n_out = (S::D3 + S::D1 + S::D2) * R;
  float* Bt = reinterpret_cast<float*>(cps4);
  float* Ct = Bt + R * S::P1;
  float* At = Ct + R * S::P2;
  float* Pst = At + R * S::P3;            // [R][68] s (*) t
  float* Pqt = Pst + R * kCpItemStride;    // [R][68] q (*) t
  float* Pqs = Pqt + R * kCpItemStride;    // [R][68] q (*) s
  float* Xs = Pqs + R * kCpItemStride;     // [D1][68] x
  float* Ys = Xs + S::D1 * kCpItemStride;  // [D2][68] y
  float* Gs = Ys + S::D2 * kCpItemStride;  // [D3][68] g_z
  float* Acc = Gs + S::D3 * kCpItemStride; // [n_out] this block's partial
  load_factors<S>(a.A, a.B, a.C, R, Bt, Ct, At);
  const int t = threadIdx.x;
  for (int o = t; o < n_out; o += T) Acc[o] = 0.f;  // entries o = t (mod 64) belong to thread t
  __syncthreads();
  const long long t0 = (long long)blockIdx.x * tpb;
  const long long t1 = t0 + tpb < tiles ? t0 + tpb : tiles;
  for (long long tile = t0; tile < t1; ++tile) {
    cp_bwd_item<S, true>(a, tile * T + t, t, Bt, Ct, At, Pst, Pqt, Pqs, Xs, Ys, Gs);
    __syncthreads();  // the tile's columns are staged
    for (int o = t; o < n_out; o += T) {
      const float* lhs;
      const float* rhs;
      if (o < S::D3 * R) {
        lhs = Gs + (o / R) * kCpItemStride;
        rhs = Pst + (o % R) * kCpItemStride;
      } else if (o < (S::D3 + S::D1) * R) {
        const int o1 = o - S::D3 * R;
        lhs = Xs + (o1 / R) * kCpItemStride;
        rhs = Pqt + (o1 % R) * kCpItemStride;
      } else {
        const int o2 = o - (S::D3 + S::D1) * R;
        lhs = Ys + (o2 / R) * kCpItemStride;
        rhs = Pqs + (o2 % R) * kCpItemStride;
      }
      float v[4] = {0.f, 0.f, 0.f, 0.f};  // four interleaved partial sums over the tile's items
#pragma unroll 4
      for (int it = 0; it < T; it += 4) {
        const float4 l4 = *reinterpret_cast<const float4*>(lhs + it);
        const float4 r4 = *reinterpret_cast<const float4*>(rhs + it);
        v[0] = fmaf(l4.x, r4.x, v[0]);
        v[1] = fmaf(l4.y, r4.y, v[1]);
        v[2] = fmaf(l4.z, r4.z, v[2]);
        v[3] = fmaf(l4.w, r4.w, v[3]);
      }
      Acc[o] += (v[0] + v[1]) + (v[2] + v[3]);
    }
    __syncthreads();  // the tile's columns are consumed
  }
  float* part = a.partial + (long long)blockIdx.x * n_out;
  for (int o = t; o < n_out; o += T) part[o] = Acc[o];
}

// g_A, g_B, g_C = the sum of the block partials.  A block of 256 threads takes
// 32 entries: warp w sums the partials k = w (mod 8) in increasing k, then
// warp 0 adds the eight warp sums in warp order.
constexpr int kCpRedEntries = 32, kCpRedWarps = 8;
__global__ void __launch_bounds__(32 * kCpRedWarps)
    cp_reduce_kernel(int blocks, int d1, int d2, int d3, int R, const float* __restrict__ partial,
                     float* __restrict__ gA, float* __restrict__ gB, float* __restrict__ gC) {
  __shared__ float part[kCpRedWarps][kCpRedEntries];
  const int n_out = (d1 + d2 + d3) * R;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int o = blockIdx.x * kCpRedEntries + lane;
  float v = 0.f;
  if (o < n_out) {
    int k = w;
    for (; k + 7 * kCpRedWarps < blocks; k += 8 * kCpRedWarps) {  // eight loads in flight, added in k order
      float q[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) q[c] = partial[(long long)(k + c * kCpRedWarps) * n_out + o];
#pragma unroll
      for (int c = 0; c < 8; ++c) v += q[c];
    }
    for (; k < blocks; k += kCpRedWarps) v += partial[(long long)k * n_out + o];
  }
  part[w][lane] = v;
  __syncthreads();
  if (w == 0 && o < n_out) {
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < kCpRedWarps; ++q) s += part[q][lane];
    if (o < d3 * R) {
      if (gA) gA[o] = s;
    } else if (o < (d3 + d1) * R) {
      if (gB) gB[o - d3 * R] = s;
    } else {
      if (gC) gC[o - (d3 + d1) * R] = s;
    }
  }
}

}  // namespace

template <int LI, int LS, int LO>
size_t cp_smem_bytes(int rank, bool factor_grads) {
  using S = CpShape<LI, LS, LO>;
  size_t n = (size_t)rank * S::PT;
  if (factor_grads)
    n += (size_t)(3 * rank + S::D1 + S::D2 + S::D3) * kCpItemStride + (size_t)(S::D1 + S::D2 + S::D3) * rank;
  return sizeof(float) * n;
}

template <int LI, int LS, int LO>
cudaError_t launch_cp_fwd(const CPArgs& a, cudaStream_t stream) {
  using S = CpShape<LI, LS, LO>;
  const long long items = (long long)a.batch * a.mult;
  if (items == 0) return cudaSuccess;
  const size_t smem = cp_smem_bytes<LI, LS, LO>(a.rank, false);
  cudaError_t e = cudaFuncSetAttribute(cp_fwd_kernel<S>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cp_fwd_kernel<S><<<(unsigned)((items + kCpFwdThreads - 1) / kCpFwdThreads), kCpFwdThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

template <int LI, int LS, int LO>
cudaError_t launch_cp_bwd(const CPArgs& a, cudaStream_t stream) {
  using S = CpShape<LI, LS, LO>;
  const long long items = (long long)a.batch * a.mult;
  const bool gf = a.grad_A != nullptr || a.grad_B != nullptr || a.grad_C != nullptr;
  const size_t smem = cp_smem_bytes<LI, LS, LO>(a.rank, gf);
  cudaError_t e;
  if (gf) {
    if (items > 0) {
      e = cudaFuncSetAttribute(cp_bwd_factors_kernel<S>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      cp_bwd_factors_kernel<S><<<(unsigned)cp_bwd_blocks(a.batch, a.mult), kCpBwdItems, smem, stream>>>(
          a, cp_bwd_tiles(a.batch, a.mult), cp_bwd_tiles_per_block(a.batch, a.mult));
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    // also for an empty batch: the gradients are then zero
    const int n_out = (S::D1 + S::D2 + S::D3) * a.rank;
    const int blocks = items > 0 ? (int)cp_bwd_blocks(a.batch, a.mult) : 0;
    cp_reduce_kernel<<<(n_out + kCpRedEntries - 1) / kCpRedEntries, 32 * kCpRedWarps, 0, stream>>>(
        blocks, S::D1, S::D2, S::D3, a.rank, a.partial, a.grad_A, a.grad_B, a.grad_C);
    return cudaGetLastError();
  }
  if (items == 0 || (a.grad_x == nullptr && a.grad_y == nullptr)) return cudaSuccess;
  e = cudaFuncSetAttribute(cp_bwd_kernel<S>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cp_bwd_kernel<S><<<(unsigned)((items + kCpBwdThreads - 1) / kCpBwdThreads), kCpBwdThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

// One translation unit per shape (the build passes CGTP_CFG_LI/LS/LO).
template size_t cp_smem_bytes<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(int, bool);
template cudaError_t launch_cp_fwd<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(const CPArgs&, cudaStream_t);
template cudaError_t launch_cp_bwd<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(const CPArgs&, cudaStream_t);

}  // namespace cgtp
