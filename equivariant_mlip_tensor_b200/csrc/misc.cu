// Per-atom forces from edge gradients, materialised spherical harmonics, and
// the row gather / scatter-add of the domain decomposition's halo exchange,
// for sm_100a.
//
// Forces: with r_e = pos_src - pos_dst, dE/dpos_n = sum_{e: src=n} g_e -
// sum_{e: dst=n} g_e and F = -dE/dpos; each node sums its CSR row
// (contiguous) and its CSC row (through the edge permutation), so there are
// no atomics and the summation order is fixed.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace cgtp {
CGTP_DEFINE_CONSTANT_TABLES()
}  // namespace cgtp

#include "sh.cuh"

namespace cgtp {
namespace {

__global__ void forces_kernel(int n, const int* __restrict__ row_ptr, const int* __restrict__ csc_ptr,
                              const int* __restrict__ csc_edge, const float* __restrict__ g,
                              float* __restrict__ F) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    float fx = 0.f, fy = 0.f, fz = 0.f;
    for (int e = row_ptr[i]; e < row_ptr[i + 1]; ++e) {
      fx += g[3 * (long long)e];
      fy += g[3 * (long long)e + 1];
      fz += g[3 * (long long)e + 2];
    }
    for (int k = csc_ptr[i]; k < csc_ptr[i + 1]; ++k) {
      const long long e = csc_edge[k];
      fx -= g[3 * e];
      fy -= g[3 * e + 1];
      fz -= g[3 * e + 2];
    }
    F[3 * i] = fx;
    F[3 * i + 1] = fy;
    F[3 * i + 2] = fz;
  }
}

template <int LS>
__global__ void sh_kernel(int n_edges, const float* __restrict__ ev, float* __restrict__ Y, float* __restrict__ dY) {
  constexpr int NS = (LS + 1) * (LS + 1);
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n_edges;
       e += (long long)gridDim.x * blockDim.x) {
    if (dY == nullptr) {
      float y[NS];
      sh_of_vec<LS>(ev[3 * e], ev[3 * e + 1], ev[3 * e + 2], y);
#pragma unroll
      for (int b = 0; b < NS; ++b) Y[e * NS + b] = y[b];
    } else {
      Dual3 y[NS];
      sh_grad_of_vec<LS>(ev[3 * e], ev[3 * e + 1], ev[3 * e + 2], y);
#pragma unroll
      for (int b = 0; b < NS; ++b) {
        if (Y) Y[e * NS + b] = y[b].v;
        dY[(e * NS + b) * 3] = y[b].d0;
        dY[(e * NS + b) * 3 + 1] = y[b].d1;
        dY[(e * NS + b) * 3 + 2] = y[b].d2;
      }
    }
  }
}

// u[e] = (dY_e/dr_e) q[e]: the harmonics' derivative along a per-edge direction.
template <int LS>
__global__ void sh_dir_kernel(int n_edges, const float* __restrict__ ev, const float* __restrict__ q,
                              float* __restrict__ u) {
  constexpr int NS = (LS + 1) * (LS + 1);
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n_edges;
       e += (long long)gridDim.x * blockDim.x) {
    Dual1 y[NS];
    sh_dir_of_vec<LS>(ev[3 * e], ev[3 * e + 1], ev[3 * e + 2], q[3 * e], q[3 * e + 1], q[3 * e + 2], y);
#pragma unroll
    for (int b = 0; b < NS; ++b) u[e * NS + b] = y[b].e;
  }
}

// Row gather and scatter-add (the pack and unpack of a halo exchange):
// element t of the n x rf block is row t / rf, column t % rf; float4 steps
// when every row is a whole number of 16-byte vectors.
__global__ void gather_rows_kernel(long long total, int rf, int vec4, const int* __restrict__ idx,
                                   const float* __restrict__ src, float* __restrict__ dst) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  if (vec4) {
    const int rq = rf / 4;
    for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < total / 4; t += stride) {
      const long long r = t / rq, c = t % rq;
      reinterpret_cast<float4*>(dst)[r * rq + c] = reinterpret_cast<const float4*>(src)[(long long)idx[r] * rq + c];
    }
  } else {
    for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < total; t += stride) {
      const long long r = t / rf, c = t % rf;
      dst[r * rf + c] = src[(long long)idx[r] * rf + c];
    }
  }
}

__global__ void scatter_add_rows_kernel(long long total, int rf, int vec4, const int* __restrict__ idx,
                                        const float* __restrict__ src, float* __restrict__ dst) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  if (vec4) {
    const int rq = rf / 4;
    for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < total / 4; t += stride) {
      const long long r = t / rq, c = t % rq;
      float4* d = reinterpret_cast<float4*>(dst) + (long long)idx[r] * rq + c;
      const float4 v = reinterpret_cast<const float4*>(src)[r * rq + c];
      float4 o = *d;
      o.x += v.x;
      o.y += v.y;
      o.z += v.z;
      o.w += v.w;
      *d = o;
    }
  } else {
    for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < total; t += stride) {
      const long long r = t / rf, c = t % rf;
      dst[(long long)idx[r] * rf + c] += src[r * rf + c];
    }
  }
}

}  // namespace

cudaError_t launch_rows(bool add, int n, int rf, const int* idx, const float* src, float* dst, int num_sms,
                        cudaStream_t stream) {
  if (n == 0 || rf == 0) return cudaSuccess;
  const long long total = (long long)n * rf;
  const int vec4 = (rf % 4 == 0 && ((uintptr_t)src & 15u) == 0 && ((uintptr_t)dst & 15u) == 0) ? 1 : 0;
  long long b = ((vec4 ? total / 4 : total) + 255) / 256;
  if (b > num_sms * 16LL) b = num_sms * 16LL;
  if (add) scatter_add_rows_kernel<<<(int)b, 256, 0, stream>>>(total, rf, vec4, idx, src, dst);
  else gather_rows_kernel<<<(int)b, 256, 0, stream>>>(total, rf, vec4, idx, src, dst);
  return cudaGetLastError();
}

cudaError_t launch_sh_dir(int lmax_sh, int n_edges, const float* ev, const float* q, float* u, int num_sms,
                          cudaStream_t stream) {
  if (n_edges == 0) return cudaSuccess;
  long long b = ((long long)n_edges + 127) / 128;
  if (b > num_sms * 16LL) b = num_sms * 16LL;
  switch (lmax_sh) {
    case 0: sh_dir_kernel<0><<<(int)b, 128, 0, stream>>>(n_edges, ev, q, u); break;
    case 1: sh_dir_kernel<1><<<(int)b, 128, 0, stream>>>(n_edges, ev, q, u); break;
    case 2: sh_dir_kernel<2><<<(int)b, 128, 0, stream>>>(n_edges, ev, q, u); break;
    case 3: sh_dir_kernel<3><<<(int)b, 128, 0, stream>>>(n_edges, ev, q, u); break;
    case 4: sh_dir_kernel<4><<<(int)b, 128, 0, stream>>>(n_edges, ev, q, u); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_forces(int n, const int* row_ptr, const int* csc_ptr, const int* csc_edge, const float* g,
                          float* F, int num_sms, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  long long b = ((long long)n + 127) / 128;
  if (b > num_sms * 16LL) b = num_sms * 16LL;
  forces_kernel<<<(int)b, 128, 0, stream>>>(n, row_ptr, csc_ptr, csc_edge, g, F);
  return cudaGetLastError();
}

cudaError_t launch_sh(int lmax_sh, int n_edges, const float* ev, float* Y, float* dY, int num_sms,
                      cudaStream_t stream) {
  if (n_edges == 0) return cudaSuccess;
  long long b = ((long long)n_edges + 127) / 128;
  if (b > num_sms * 16LL) b = num_sms * 16LL;
  switch (lmax_sh) {
    case 0: sh_kernel<0><<<(int)b, 128, 0, stream>>>(n_edges, ev, Y, dY); break;
    case 1: sh_kernel<1><<<(int)b, 128, 0, stream>>>(n_edges, ev, Y, dY); break;
    case 2: sh_kernel<2><<<(int)b, 128, 0, stream>>>(n_edges, ev, Y, dY); break;
    case 3: sh_kernel<3><<<(int)b, 128, 0, stream>>>(n_edges, ev, Y, dY); break;
    case 4: sh_kernel<4><<<(int)b, 128, 0, stream>>>(n_edges, ev, Y, dY); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace cgtp
