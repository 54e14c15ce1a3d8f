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
// each block of 64 (pair, channel) items stages its per-item rank vectors
// (s (*) t, q (*) t, q (*) s) and inputs in shared memory, contracts them over
// its items into one partial of every factor entry, and a second kernel sums
// the block partials in block order (bit-reproducible).
#include "common.cuh"
#include "launch.h"

namespace cgtp {
namespace {

constexpr int kCpFwdThreads = 128;
constexpr int kCpBwdItems = kCpItemsPerPartial;  // items (and threads) per backward block with factor gradients
constexpr int kCpBwdThreads = 128;
constexpr int kCpItemStride = kCpBwdItems + 1;  // staged rows padded against bank conflicts

constexpr int pad4(int d) { return (d + 3) & ~3; }

template <int LI, int LS, int LO>
struct CpShape {
  static constexpr int D1 = (LI + 1) * (LI + 1), D2 = (LS + 1) * (LS + 1), D3 = (LO + 1) * (LO + 1);
  static constexpr int P1 = pad4(D1), P2 = pad4(D2), P3 = pad4(D3);
  static constexpr int PT = P1 + P2 + P3;  // transposed factor floats per rank component
};

// Factors into shared memory as [r][row] with rows padded by zeros.
template <class S>
__device__ __forceinline__ void load_factors(const float* __restrict__ A, const float* __restrict__ B,
                                             const float* __restrict__ C, int R, float* Bt, float* Ct, float* At) {
  for (int idx = threadIdx.x; idx < R * S::PT; idx += blockDim.x) {
    const int r = idx / S::PT, c = idx % S::PT;
    float v = 0.f;
    if (c < S::P1) {
      if (c < S::D1) v = B[c * R + r];
      Bt[r * S::P1 + c] = v;
    } else if (c < S::P1 + S::P2) {
      const int j = c - S::P1;
      if (j < S::D2) v = C[j * R + r];
      Ct[r * S::P2 + j] = v;
    } else {
      const int k = c - S::P1 - S::P2;
      if (k < S::D3) v = A[k * R + r];
      At[r * S::P3 + k] = v;
    }
  }
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

// Backward.  GF: also the block partials of the factor gradients.
template <class S, bool GF>
__global__ void __launch_bounds__(GF ? kCpBwdItems : kCpBwdThreads) cp_bwd_kernel(CPArgs a) {
  constexpr int T = GF ? kCpBwdItems : kCpBwdThreads;
  extern __shared__ float4 cps4[];
  float* Bt = reinterpret_cast<float*>(cps4);
  float* Ct = Bt + a.rank * S::P1;
  float* At = Ct + a.rank * S::P2;
  float* Pst = At + a.rank * S::P3;             // GF: [R][65] s (*) t
  float* Pqt = Pst + a.rank * kCpItemStride;     // GF: [R][65] q (*) t
  float* Pqs = Pqt + a.rank * kCpItemStride;     // GF: [R][65] q (*) s
  float* Xs = Pqs + a.rank * kCpItemStride;      // GF: [D1][65] x
  float* Ys = Xs + S::D1 * kCpItemStride;        // GF: [D2][65] y
  float* Gs = Ys + S::D2 * kCpItemStride;        // GF: [D3][65] g_z
  load_factors<S>(a.A, a.B, a.C, a.rank, Bt, Ct, At);
  __syncthreads();
  const int t = threadIdx.x;
  const long long item = (long long)blockIdx.x * T + t;
  const long long items = (long long)a.batch * a.mult;
  const bool ok = item < items;
  if (!GF && !ok) return;
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
    __syncthreads();
    // block partial of every factor entry: [g_A (D3 x R) | g_B (D1 x R) | g_C (D2 x R)]
    const int R = a.rank;
    const int n_out = (S::D3 + S::D1 + S::D2) * R;
    float* part = a.partial + (long long)blockIdx.x * n_out;
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
      float v = 0.f;
#pragma unroll 8
      for (int it = 0; it < T; ++it) v = fmaf(lhs[it], rhs[it], v);
      part[o] = v;
    }
  }
}

// g_A, g_B, g_C = the block partials summed in block order.
__global__ void cp_reduce_kernel(int blocks, int d1, int d2, int d3, int R, const float* __restrict__ partial,
                                 float* __restrict__ gA, float* __restrict__ gB, float* __restrict__ gC) {
  const int n_out = (d1 + d2 + d3) * R;
  for (int o = blockIdx.x * blockDim.x + threadIdx.x; o < n_out; o += gridDim.x * blockDim.x) {
    float v = 0.f;
    for (int k = 0; k < blocks; ++k) v += partial[(long long)k * n_out + o];
    if (o < d3 * R) {
      if (gA) gA[o] = v;
    } else if (o < (d3 + d1) * R) {
      if (gB) gB[o - d3 * R] = v;
    } else {
      if (gC) gC[o - (d3 + d1) * R] = v;
    }
  }
}

}  // namespace

template <int LI, int LS, int LO>
size_t cp_smem_bytes(int rank, bool factor_grads) {
  using S = CpShape<LI, LS, LO>;
  size_t n = (size_t)rank * S::PT;
  if (factor_grads) n += (size_t)(3 * rank + S::D1 + S::D2 + S::D3) * kCpItemStride;
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
  if (items > 0 && (gf || a.grad_x != nullptr || a.grad_y != nullptr)) {
    const size_t smem = cp_smem_bytes<LI, LS, LO>(a.rank, gf);
    cudaError_t e;
    if (gf) {
      e = cudaFuncSetAttribute(cp_bwd_kernel<S, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      cp_bwd_kernel<S, true><<<(unsigned)cp_bwd_blocks(a.batch, a.mult), kCpBwdItems, smem, stream>>>(a);
    } else {
      e = cudaFuncSetAttribute(cp_bwd_kernel<S, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      cp_bwd_kernel<S, false>
          <<<(unsigned)((items + kCpBwdThreads - 1) / kCpBwdThreads), kCpBwdThreads, smem, stream>>>(a);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (gf) {  // also for an empty batch: the gradients are then zero
    const int n_out = (S::D1 + S::D2 + S::D3) * a.rank;
    cp_reduce_kernel<<<(n_out + 255) / 256, 256, 0, stream>>>((int)cp_bwd_blocks(a.batch, a.mult), S::D1, S::D2,
                                                             S::D3, a.rank, a.partial, a.grad_A, a.grad_B,
                                                             a.grad_C);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

// One translation unit per shape (the build passes CGTP_CFG_LI/LS/LO).
template size_t cp_smem_bytes<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(int, bool);
template cudaError_t launch_cp_fwd<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(const CPArgs&, cudaStream_t);
template cudaError_t launch_cp_bwd<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(const CPArgs&, cudaStream_t);

}  // namespace cgtp
