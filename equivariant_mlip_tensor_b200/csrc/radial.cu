// Radial weight network for sm_100a: per-edge, per-path, per-channel weights
// W_e = SiLU(phi(|r_e|) W1) W2 and the derivative of a loss through them.
//
// phi_k(r) = exp(-(r - mu_k)^2 / (2 sigma^2)), mu_k = k rc / 7, sigma = rc / 7
// (k = 0..7), W1 [8][64], W2 [64][P*mult], no biases.  The convolution
// scales each path by these weights ("LunaTP ...", abstract); the network
// itself is the synthetic workloads' weight generator.
//
// Forward: a GEMM with K = 64 and 128 x 128 output tiles.  Persistent blocks
// (two per SM) take contiguous ranges of tiles in edge-tile-major order, keep
// the hidden layer of the current 128 edges in shared memory (k-major), and
// copy the next tile's 64 x 128 slice of W2 (cp.async, double-buffered) while
// each thread accumulates an 8 x 8 register tile in fp32.
// The forward's 8 x 8 tiles use the packed f32x2 FMA (two lanes of fp32 per
// instruction, rounded like two fmaf), which halves the issue slots the
// products take.
// Backward: grad_h = grad_W W2^T is a GEMM with M = edges, N = 64, K = P*mult;
// each block owns 96 edges and all 64 hidden units, streams grad_W once
// through a two-stage cp.async pipeline, and its epilogue folds grad_h
// through SiLU', W1 and dphi/dr into dL/d|r| per edge, added to
// grad_edge_vec along r/|r| (one owner per edge, no atomics).
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

// Asynchronous 16-byte global -> shared copies (cp.async, bypassing L1).
// src_bytes = 0 writes zeros and reads nothing, which pads ragged tiles.
static __device__ __forceinline__ void cp16(float* dst, const float* src, int src_bytes) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(src_bytes) : "memory");
}
static __device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
static __device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------- forward
constexpr int kFwdBM = 128, kFwdBN = 128, kFwdThreads = 256;
constexpr int kFwdSmem = sizeof(float) * (kRH * kFwdBM + 2 * kRH * kFwdBN);  // Hs + two W2 stages

// Work units are (128-edge tile, 128-output tile) pairs in edge-tile-major order;
// a persistent block takes a contiguous range of them, so it evaluates the
// hidden layer only when its edge tile changes, and the W2 slice of the next
// unit is copied (cp.async) while the current one is multiplied.
static __global__ void __launch_bounds__(kFwdThreads, 2)
    radial_fwd_kernel(int n_edges, int N, long long n_units, const float* __restrict__ ev, float rc,
                      const float* __restrict__ W1, const float* __restrict__ W2, float* __restrict__ w) {
  extern __shared__ float4 rsm4[];
  float* Hs = reinterpret_cast<float*>(rsm4);  // [64][128] k-major
  float* Bs = Hs + kRH * kFwdBM;               // 2 x [64][128]
  const int t = threadIdx.x;
  const int n_nt = (N + kFwdBN - 1) / kFwdBN;
  const long long u0 = (long long)blockIdx.x * n_units / gridDim.x;
  const long long u1 = (long long)(blockIdx.x + 1) * n_units / gridDim.x;
  auto stage_w2 = [&](long long u, int s) {  // W2[:, n0 .. n0+128) -> stage s
    const int n0 = (int)(u % n_nt) * kFwdBN;
    float* dst = Bs + s * (kRH * kFwdBN);
#pragma unroll
    for (int q = 0; q < kRH * kFwdBN / 4 / kFwdThreads; ++q) {
      const int idx = t + kFwdThreads * q;
      const int k = idx / (kFwdBN / 4), n4 = idx % (kFwdBN / 4);
      const int n = n0 + 4 * n4;
      const bool ok = n < N;
      cp16(dst + k * kFwdBN + 4 * n4, ok ? W2 + (long long)k * N + n : W2, ok ? 16 : 0);
    }
    cp_commit();
  };
  if (u0 < u1) stage_w2(u0, 0);
  long long cur_mt = -1;
  const int tx = t & 15, ty = t >> 4;
  for (long long u = u0; u < u1; ++u) {
    const int s = (int)((u - u0) & 1);
    const long long mt = u / n_nt;
    const int n0 = (int)(u % n_nt) * kFwdBN;
    const long long m0 = mt * kFwdBM;
    __syncthreads();  // the previous unit's reads of Hs and of stage s^1 are done
    if (u + 1 < u1) stage_w2(u + 1, s ^ 1);
    if (mt != cur_mt) {  // hidden layer of the tile's edges: thread -> (edge, half of the hidden units)
      cur_mt = mt;
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
    if (u + 1 < u1)
      cp_wait<1>();
    else
      cp_wait<0>();
    __syncthreads();  // stage s and Hs are visible to every thread
    const float* B = Bs + s * (kRH * kFwdBN);
    float2 acc[8][4];  // (acc[i][2p], acc[i][2p + 1]) packed for the f32x2 FMA
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int p = 0; p < 4; ++p) acc[i][p] = make_float2(0.f, 0.f);
#pragma unroll 8
    for (int k = 0; k < kRH; ++k) {
      const float4 a0 = reinterpret_cast<const float4*>(Hs + k * kFwdBM + ty * 8)[0];
      const float4 a1 = reinterpret_cast<const float4*>(Hs + k * kFwdBM + ty * 8)[1];
      const float4 b0 = reinterpret_cast<const float4*>(B + k * kFwdBN)[tx];
      const float4 b1 = reinterpret_cast<const float4*>(B + k * kFwdBN)[16 + tx];
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float2 bp[4] = {make_float2(b0.x, b0.y), make_float2(b0.z, b0.w), make_float2(b1.x, b1.y),
                            make_float2(b1.z, b1.w)};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 ad = make_float2(av[i], av[i]);
#pragma unroll
        for (int p = 0; p < 4; ++p) acc[i][p] = __ffma2_rn(ad, bp[p], acc[i][p]);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const long long e = m0 + ty * 8 + i;
      if (e < n_edges) {
        float* row = w + e * N;
        const int na = n0 + 4 * tx, nb = n0 + 64 + 4 * tx;
        if (na < N)
          *reinterpret_cast<float4*>(row + na) = make_float4(acc[i][0].x, acc[i][0].y, acc[i][1].x, acc[i][1].y);
        if (nb < N)
          *reinterpret_cast<float4*>(row + nb) = make_float4(acc[i][2].x, acc[i][2].y, acc[i][3].x, acc[i][3].y);
      }
    }
  }
}

cudaError_t launch_radial_fwd(int n_edges, int N, const float* ev, float rc, const float* W1, const float* W2,
                              float* w, int num_sms, cudaStream_t stream) {
  if (n_edges == 0 || N == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(radial_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFwdSmem);
  if (e != cudaSuccess) return e;
  const long long units = ((long long)n_edges + kFwdBM - 1) / kFwdBM * ((N + kFwdBN - 1) / kFwdBN);
  const long long grid = units < 2LL * num_sms ? units : 2LL * num_sms;
  radial_fwd_kernel<<<(unsigned)grid, kFwdThreads, kFwdSmem, stream>>>(n_edges, N, units, ev, rc, W1, W2, w);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- backward
// grad_h [96 edges][64 hidden] = grad_W [96][N] W2^T, K = N in chunks of 32
// staged by cp.async in two stages.  Shared rows are padded to 36 floats so
// that the per-thread float4 reads fall in distinct banks; thread (ty, tx)
// owns edges ty + 16 i and hidden units tx + 8 j, a 6 x 8 register tile.
// Edges per thread: 96-edge tiles (6 per thread) fill the 4 resident blocks per
// SM in 1.7 waves at 97 480 edges where 128-edge tiles leave a 1.3-wave tail
// (0.69 vs 0.76 ms measured; 112-edge tiles 0.72 ms).
constexpr int kEPT = 6;
constexpr int kBwdBM = 16 * kEPT, kBwdBK = 32, kBwdStride = kBwdBK + 4, kBwdThreads = 128;
constexpr int kBwdSmem = (int)sizeof(float) * 2 * (kBwdBM + kRH) * kBwdStride;

static __global__ void __launch_bounds__(kBwdThreads, 4)
    radial_bwd_kernel(int n_edges, int N, const float* __restrict__ ev, float rc, const float* __restrict__ W1,
                      const float* __restrict__ W2, const float* __restrict__ gw, float* __restrict__ gev) {
  extern __shared__ float4 rsm4[];
  float* As = reinterpret_cast<float*>(rsm4);  // 2 x [96][36]   grad_W chunk, [edge][n]
  float* Bs = As + 2 * kBwdBM * kBwdStride;    // 2 x [64][36]   W2 chunk, [hidden][n]
  const int t = threadIdx.x;
  const int tx = t & 7, ty = t >> 3;
  const long long m0 = (long long)blockIdx.x * kBwdBM;
  auto stage = [&](int n0, int s) {
    float* a = As + s * kBwdBM * kBwdStride;
#pragma unroll
    for (int q = 0; q < kBwdBM * 8 / kBwdThreads; ++q) {
      const int idx = t + kBwdThreads * q;
      const int m = idx >> 3, c = idx & 7;
      const long long e = m0 + m;
      const int n = n0 + 4 * c;
      const bool ok = e < n_edges && n < N;
      cp16(a + m * kBwdStride + 4 * c, ok ? gw + e * N + n : gw, ok ? 16 : 0);
    }
    float* b = Bs + s * kRH * kBwdStride;
#pragma unroll
    for (int q = 0; q < kRH * 8 / kBwdThreads; ++q) {
      const int idx = t + kBwdThreads * q;
      const int k = idx >> 3, c = idx & 7;
      const int n = n0 + 4 * c;
      const bool ok = n < N;
      cp16(b + k * kBwdStride + 4 * c, ok ? W2 + (long long)k * N + n : W2, ok ? 16 : 0);
    }
    cp_commit();
  };
  float acc[kEPT][8];
#pragma unroll
  for (int i = 0; i < kEPT; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  const int n_chunks = (N + kBwdBK - 1) / kBwdBK;
  stage(0, 0);
  for (int c = 0; c < n_chunks; ++c) {
    const int s = c & 1;
    __syncthreads();  // reads of stage s^1 (chunk c - 1) are done
    if (c + 1 < n_chunks) {
      stage((c + 1) * kBwdBK, s ^ 1);
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();  // stage s is visible to every thread
    const float* a = As + s * kBwdBM * kBwdStride;
    const float* b = Bs + s * kRH * kBwdStride;
#pragma unroll 1
    for (int q = 0; q < kBwdBK / 4; ++q) {
      float4 av[kEPT];
#pragma unroll
      for (int i = 0; i < kEPT; ++i) av[i] = *reinterpret_cast<const float4*>(a + (ty + 16 * i) * kBwdStride + 4 * q);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 bv = *reinterpret_cast<const float4*>(b + (tx + 8 * j) * kBwdStride + 4 * q);
#pragma unroll
        for (int i = 0; i < kEPT; ++i) {
          acc[i][j] = fmaf(av[i].x, bv.x, acc[i][j]);
          acc[i][j] = fmaf(av[i].y, bv.y, acc[i][j]);
          acc[i][j] = fmaf(av[i].z, bv.z, acc[i][j]);
          acc[i][j] = fmaf(av[i].w, bv.w, acc[i][j]);
        }
      }
    }
  }
  // epilogue: dL/dr = sum_k grad_h[k] SiLU'(a_k) (dphi W1)_k, per edge
#pragma unroll
  for (int i = 0; i < kEPT; ++i) {
    const long long e = m0 + ty + 16 * i;
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
    for (int j = 0; j < 8; ++j) {
      const int k = tx + 8 * j;
      float av = 0.f, bv = 0.f;
#pragma unroll
      for (int q = 0; q < kRB; ++q) {
        const float w1 = __ldg(W1 + q * kRH + k);
        av = fmaf(phi[q], w1, av);
        bv = fmaf(dphi[q], w1, bv);
      }
      const float sg = 1.f / (1.f + expf(-av));
      const float ds = sg * (1.f + av * (1.f - sg));
      part = fmaf(acc[i][j] * ds, bv, part);
    }
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (tx == 0 && e < n_edges && r > 0.f) {
      const float sc = part / r;
      gev[3 * e] += sc * x;
      gev[3 * e + 1] += sc * y;
      gev[3 * e + 2] += sc * z;
    }
  }
}

cudaError_t launch_radial_bwd(int n_edges, int N, const float* ev, float rc, const float* W1, const float* W2,
                              const float* gw, float* gev, int num_sms, cudaStream_t stream) {
  (void)num_sms;
  if (n_edges == 0 || N == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(radial_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kBwdSmem);
  if (e != cudaSuccess) return e;
  radial_bwd_kernel<<<(unsigned)((n_edges + kBwdBM - 1) / kBwdBM), kBwdThreads, kBwdSmem, stream>>>(
      n_edges, N, ev, rc, W1, W2, gw, gev);
  return cudaGetLastError();
}

}  // namespace cgtp
