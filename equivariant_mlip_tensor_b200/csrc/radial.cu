// Radial weight network for sm_100a: per-edge, per-path, per-channel weights
// W_e = SiLU(phi(|r_e|) W1) W2 and the derivative of a loss through them.
//
// phi_k(r) = exp(-(r - mu_k)^2 / (2 sigma^2)), mu_k = k rc / 7, sigma = rc / 7
// (k = 0..7), W1 [8][64], W2 [64][P*mult], no biases.  The convolution
// scales each path by these weights ("LunaTP ...", abstract); the network
// itself is the synthetic workloads' weight generator.
//
// Forward: a GEMM with K = 64.  Each block owns a 128-edge x 128-output
// tile row: it evaluates the hidden layer of its 128 edges once into shared
// memory (k-major), then for every 128-wide output tile stages the 64 x 128
// slice of W2 and each thread accumulates an 8 x 8 register tile in fp32
// (four 128-bit shared loads per 64 FMAs).
// Backward: grad_h = grad_W W2^T is a GEMM with M = edges, N = 64, K = P*mult;
// each block owns 64 edges and all 64 hidden units, streams grad_W once, and
// its epilogue folds grad_h through SiLU', W1 and dphi/dr into
// dL/d|r| per edge, added to grad_edge_vec along r/|r| (one owner per edge,
// no atomics).
#include <cuda_runtime.h>

#include "common.cuh"

namespace cgtp {

constexpr int kRB = 8;   // Gaussian basis size
constexpr int kRH = 64;  // hidden units

static __device__ __forceinline__ void radial_basis(float r, float rc, float (&phi)[kRB], float (&dphi)[kRB]) {
  const float sigma = rc / float(kRB - 1);
  const float inv2s2 = 1.f / (2.f * sigma * sigma);
#pragma unroll
  for (int k = 0; k < kRB; ++k) {
    const float d = r - float(k) * sigma;
    phi[k] = expf(-d * d * inv2s2);
    dphi[k] = -2.f * d * inv2s2 * phi[k];
  }
}

// ---------------------------------------------------------------- forward
constexpr int kFwdBM = 128, kFwdBN = 128;

static __global__ void __launch_bounds__(256) radial_fwd_kernel(int n_edges, int N, const float* __restrict__ ev,
                                                         float rc, const float* __restrict__ W1,
                                                         const float* __restrict__ W2, float* __restrict__ w) {
  extern __shared__ float4 rsm4[];
  float* Hs = reinterpret_cast<float*>(rsm4);  // [64][128] k-major
  float* Bs = Hs + kRH * kFwdBM;               // [64][128]
  const int t = threadIdx.x;
  const long long m0 = (long long)blockIdx.x * kFwdBM;
  {  // hidden layer of the block's edges: thread -> (edge, half of the hidden units)
    const int m = t & (kFwdBM - 1), kh = t >> 7;
    const long long e = m0 + m;
    float r = 0.f;
    if (e < n_edges) {
      const float x = ev[3 * e], y = ev[3 * e + 1], z = ev[3 * e + 2];
      r = sqrtf(fmaf(x, x, fmaf(y, y, z * z)));
    }
    float phi[kRB], dphi[kRB];
    radial_basis(r, rc, phi, dphi);
#pragma unroll 4
    for (int kk = 0; kk < kRH / 2; ++kk) {
      const int k = kh * (kRH / 2) + kk;
      float a = 0.f;
#pragma unroll
      for (int j = 0; j < kRB; ++j) a = fmaf(phi[j], __ldg(W1 + j * kRH + k), a);
      Hs[k * kFwdBM + m] = a / (1.f + expf(-a));
    }
  }
  const int tx = t & 15, ty = t >> 4;
  for (int n0 = 0; n0 < N; n0 += kFwdBN) {
    __syncthreads();  // Hs complete / previous tile's Bs reads done
    for (int idx = t; idx < kRH * kFwdBN / 4; idx += 256) {  // W2 slice [64][n0 .. n0+128)
      const int k = idx / (kFwdBN / 4), n4 = idx % (kFwdBN / 4);
      const int n = n0 + 4 * n4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (n < N) v = __ldg(reinterpret_cast<const float4*>(W2 + (long long)k * N + n));
      reinterpret_cast<float4*>(Bs + k * kFwdBN)[n4] = v;
    }
    __syncthreads();
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
#pragma unroll 8
    for (int k = 0; k < kRH; ++k) {
      const float4 a0 = reinterpret_cast<const float4*>(Hs + k * kFwdBM + ty * 8)[0];
      const float4 a1 = reinterpret_cast<const float4*>(Hs + k * kFwdBM + ty * 8)[1];
      const float4 b0 = reinterpret_cast<const float4*>(Bs + k * kFwdBN)[tx];
      const float4 b1 = reinterpret_cast<const float4*>(Bs + k * kFwdBN)[16 + tx];
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const long long e = m0 + ty * 8 + i;
      if (e < n_edges) {
        float* row = w + e * N;
        const int na = n0 + 4 * tx, nb = n0 + 64 + 4 * tx;
        if (na < N) *reinterpret_cast<float4*>(row + na) = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
        if (nb < N) *reinterpret_cast<float4*>(row + nb) = make_float4(acc[i][4], acc[i][5], acc[i][6], acc[i][7]);
      }
    }
  }
}

cudaError_t launch_radial_fwd(int n_edges, int N, const float* ev, float rc, const float* W1, const float* W2,
                              float* w, cudaStream_t stream) {
  if (n_edges == 0) return cudaSuccess;
  const size_t smem = sizeof(float) * (kRH * kFwdBM + kRH * kFwdBN);
  cudaError_t e = cudaFuncSetAttribute(radial_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  radial_fwd_kernel<<<(unsigned)((n_edges + kFwdBM - 1) / kFwdBM), 256, smem, stream>>>(n_edges, N, ev, rc, W1, W2, w);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- backward
constexpr int kBwdBM = 64, kBwdBK = 32;
constexpr int kAStride = kBwdBM + 4;

static __global__ void __launch_bounds__(128) radial_bwd_kernel(int n_edges, int N, const float* __restrict__ ev,
                                                         float rc, const float* __restrict__ W1,
                                                         const float* __restrict__ W2,
                                                         const float* __restrict__ gw,
                                                         float* __restrict__ gev) {
  __shared__ __align__(16) float As[kBwdBK][kAStride];  // grad_W chunk, [n][edge]
  __shared__ __align__(16) float Bs[kBwdBK][kRH + 4];   // W2 chunk, [n][hidden]
  const int t = threadIdx.x;
  const int tx = t & 15, ty = t >> 4;  // hidden 4*tx..+4, edges 8*ty..+8
  const long long m0 = (long long)blockIdx.x * kBwdBM;
  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  float4 pa[4], pb[4];
  auto load_chunk = [&](int n0) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int idx = t + 128 * q;  // 512 float4 of A: 64 edges x 8 float4
      const int m = idx >> 3, n4 = idx & 7;
      const long long e = m0 + m;
      const int n = n0 + 4 * n4;
      pa[q] = (e < n_edges && n < N) ? __ldcs(reinterpret_cast<const float4*>(gw + e * N + n))
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
      const int k = idx >> 3;  // 512 float4 of B: 64 hidden x 8 float4
      pb[q] = n < N ? __ldg(reinterpret_cast<const float4*>(W2 + (long long)k * N + n))
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto store_chunk = [&]() {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int idx = t + 128 * q;
      const int m = idx >> 3, n4 = idx & 7;
      As[4 * n4 + 0][m] = pa[q].x;
      As[4 * n4 + 1][m] = pa[q].y;
      As[4 * n4 + 2][m] = pa[q].z;
      As[4 * n4 + 3][m] = pa[q].w;
      Bs[4 * n4 + 0][m] = pb[q].x;
      Bs[4 * n4 + 1][m] = pb[q].y;
      Bs[4 * n4 + 2][m] = pb[q].z;
      Bs[4 * n4 + 3][m] = pb[q].w;
    }
  };
  load_chunk(0);
  for (int n0 = 0; n0 < N; n0 += kBwdBK) {
    __syncthreads();
    store_chunk();
    __syncthreads();
    if (n0 + kBwdBK < N) load_chunk(n0 + kBwdBK);
#pragma unroll 8
    for (int n = 0; n < kBwdBK; ++n) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[n][ty * 8]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[n][ty * 8 + 4]);
      const float4 b = *reinterpret_cast<const float4*>(&Bs[n][tx * 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
  }
  // epilogue: dL/dr = sum_k grad_h[k] SiLU'(a_k) (dphi W1)_k, per edge
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const long long e = m0 + ty * 8 + i;
    float x = 0.f, y = 0.f, z = 0.f, r = 0.f;
    if (e < n_edges) {
      x = ev[3 * e];
      y = ev[3 * e + 1];
      z = ev[3 * e + 2];
      r = sqrtf(fmaf(x, x, fmaf(y, y, z * z)));
    }
    float phi[kRB], dphi[kRB];
    radial_basis(r, rc, phi, dphi);
    float part = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int k = 4 * tx + j;
      float a = 0.f, b = 0.f;
#pragma unroll
      for (int q = 0; q < kRB; ++q) {
        const float w1 = __ldg(W1 + q * kRH + k);
        a = fmaf(phi[q], w1, a);
        b = fmaf(dphi[q], w1, b);
      }
      const float sg = 1.f / (1.f + expf(-a));
      const float ds = sg * (1.f + a * (1.f - sg));
      part = fmaf(acc[i][j] * ds, b, part);
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (tx == 0 && e < n_edges && r > 0.f) {
      const float s = part / r;
      gev[3 * e] += s * x;
      gev[3 * e + 1] += s * y;
      gev[3 * e + 2] += s * z;
    }
  }
}

cudaError_t launch_radial_bwd(int n_edges, int N, const float* ev, float rc, const float* W1, const float* W2,
                              const float* gw, float* gev, cudaStream_t stream) {
  if (n_edges == 0) return cudaSuccess;
  radial_bwd_kernel<<<(unsigned)((n_edges + kBwdBM - 1) / kBwdBM), 128, 0, stream>>>(n_edges, N, ev, rc, W1, W2,
                                                                                    gw, gev);
  return cudaGetLastError();
}

}  // namespace cgtp
