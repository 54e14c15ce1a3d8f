// Edge-free channelwise CG tensor product of batched pairs, for sm_100a.
//
//   z[b][l3,m3][u] = sum_p w[p][u] sum_{m1,m2} C^p[m1,m2,m3] x[b][l1,m1][u] y[b][l2,m2][u]
//
// ("Tensor Decomposition Networks ...", reply to reviewer S6y1: the exact CG
// product of two irreps inputs, timed at batch 1000 and multiplicity 128.)
// One thread per (pair, channel); consecutive threads take consecutive
// channels, so every load and store is coalesced.  The CG coefficients are
// constant-memory operands of the FMAs, unrolled over the structural
// nonzero pattern.  The backward sums grad_w over the batch in two passes
// (per-chunk partials in a workspace, then a fixed-order sum): no atomics,
// bit-reproducible.
#include "common.cuh"

namespace cgtp {
CGTP_DEFINE_CONSTANT_TABLES()
}  // namespace cgtp

namespace cgtp {


namespace {

// t[m3] = sum_{m1,m2} C x[l1,m1] y[l2,m2] for path P, folded into f(m3, t).
template <class PS, int P, class F>
__device__ __forceinline__ void path_product(const float (&xr)[PS::NI], const float (&yr)[PS::NS], F&& f) {
  constexpr int l1 = PS::D.l1[P], l2 = PS::D.l2[P], l3 = PS::D.l3[P];
  static_for<0, 2 * l3 + 1>([&](auto M3c) {
    constexpr int m3 = decltype(M3c)::value - l3;
    float t = 0.f;
    static_for<0, 2 * l1 + 1>([&](auto M1c) {
      constexpr int m1 = decltype(M1c)::value - l1;
      static_for<0, 2 * l2 + 1>([&](auto M2c) {
        constexpr int m2 = decltype(M2c)::value - l2;
        if constexpr (cg_allowed(l1, l2, l3, m1, m2, m3)) {
          t = fmaf(c_cg[table_index(l1, l2, l3, m1, m2, m3)], xr[l1 * l1 + l1 + m1] * yr[l2 * l2 + l2 + m2], t);
        }
      });
    });
    f(l3 * l3 + l3 + m3, t);
  });
}

template <class PS>
__global__ void __launch_bounds__(256) tp_fwd_kernel(TPArgs a) {
  constexpr int NI = PS::NI, NS = PS::NS, NO = PS::NO;
  const int c = blockIdx.x * 32 + threadIdx.x;
  if (c >= a.mult) return;
  for (long long b = (long long)blockIdx.y * kTpRows + threadIdx.y; b < a.batch;
       b += (long long)gridDim.y * kTpRows) {
    float xr[NI], yr[NS], z[NO];
#pragma unroll
    for (int r = 0; r < NI; ++r) xr[r] = __ldg(a.x + (b * NI + r) * a.mult + c);
#pragma unroll
    for (int r = 0; r < NS; ++r) yr[r] = __ldg(a.y + (b * NS + r) * a.mult + c);
#pragma unroll
    for (int r = 0; r < NO; ++r) z[r] = 0.f;
    static_for<0, PS::NP>([&](auto Pc) {
      constexpr int P = decltype(Pc)::value;
      const float wv = __ldg(a.w + P * a.mult + c);
      path_product<PS, P>(xr, yr, [&](int r3, float t) { z[r3] = fmaf(wv, t, z[r3]); });
    });
#pragma unroll
    for (int r = 0; r < NO; ++r) a.z[(b * NO + r) * a.mult + c] = z[r];
  }
}

template <class PS>
__global__ void __launch_bounds__(256) tp_bwd_kernel(TPArgs a) {
  constexpr int NI = PS::NI, NS = PS::NS, NO = PS::NO, NP = PS::NP;
  __shared__ float red[kTpRows][32];
  const int c = blockIdx.x * 32 + threadIdx.x;
  const bool cok = c < a.mult;
  float gwp[NP];
#pragma unroll
  for (int p = 0; p < NP; ++p) gwp[p] = 0.f;
  if (cok) {
    for (long long b = (long long)blockIdx.y * kTpRows + threadIdx.y; b < a.batch;
         b += (long long)gridDim.y * kTpRows) {
      float xr[NI], yr[NS], gr[NO], gx[NI], gy[NS];
#pragma unroll
      for (int r = 0; r < NI; ++r) { xr[r] = __ldg(a.x + (b * NI + r) * a.mult + c); gx[r] = 0.f; }
#pragma unroll
      for (int r = 0; r < NS; ++r) { yr[r] = __ldg(a.y + (b * NS + r) * a.mult + c); gy[r] = 0.f; }
#pragma unroll
      for (int r = 0; r < NO; ++r) gr[r] = __ldg(a.grad_z + (b * NO + r) * a.mult + c);
      static_for<0, NP>([&](auto Pc) {
        constexpr int P = decltype(Pc)::value;
        constexpr int l1 = PS::D.l1[P], l2 = PS::D.l2[P], l3 = PS::D.l3[P];
        const float wv = __ldg(a.w + P * a.mult + c);
        static_for<0, 2 * l3 + 1>([&](auto M3c) {
          constexpr int m3 = decltype(M3c)::value - l3;
          const float g3 = gr[l3 * l3 + l3 + m3];
          const float s = wv * g3;
          float t = 0.f;
          static_for<0, 2 * l1 + 1>([&](auto M1c) {
            constexpr int m1 = decltype(M1c)::value - l1;
            static_for<0, 2 * l2 + 1>([&](auto M2c) {
              constexpr int m2 = decltype(M2c)::value - l2;
              if constexpr (cg_allowed(l1, l2, l3, m1, m2, m3)) {
                constexpr int ci = table_index(l1, l2, l3, m1, m2, m3);
                constexpr int r1 = l1 * l1 + l1 + m1, r2 = l2 * l2 + l2 + m2;
                const float cs = c_cg[ci] * s;
                gx[r1] = fmaf(cs, yr[r2], gx[r1]);
                gy[r2] = fmaf(cs, xr[r1], gy[r2]);
                t = fmaf(c_cg[ci], xr[r1] * yr[r2], t);
              }
            });
          });
          gwp[P] = fmaf(g3, t, gwp[P]);
        });
      });
      if (a.grad_x) {
#pragma unroll
        for (int r = 0; r < NI; ++r) a.grad_x[(b * NI + r) * a.mult + c] = gx[r];
      }
      if (a.grad_y) {
#pragma unroll
        for (int r = 0; r < NS; ++r) a.grad_y[(b * NS + r) * a.mult + c] = gy[r];
      }
    }
  }
  if (a.partial == nullptr) return;  // uniform over the block
  // fixed-order sum over the block's rows, then one partial per (chunk, path, channel)
#pragma unroll 1
  for (int p = 0; p < NP; ++p) {
    red[threadIdx.y][threadIdx.x] = gwp[p];
    __syncthreads();
    if (threadIdx.y == 0 && cok) {
      float v = 0.f;
#pragma unroll
      for (int r = 0; r < kTpRows; ++r) v += red[r][threadIdx.x];
      a.partial[((long long)blockIdx.y * NP + p) * a.mult + c] = v;
    }
    __syncthreads();
  }
}

__global__ void tp_reduce_partials_kernel(int chunks, int np_mult, const float* __restrict__ partial,
                                          float* __restrict__ grad_w) {
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < np_mult; k += gridDim.x * blockDim.x) {
    float v = 0.f;
    for (int ch = 0; ch < chunks; ++ch) v += partial[(long long)ch * np_mult + k];
    grad_w[k] = v;
  }
}

}  // namespace

template <int LI, int LS, int LO>
cudaError_t launch_tp_fwd(const TPArgs& a, int num_sms, cudaStream_t stream) {
  using PS = PathSet<LI, LS, LO>;
  (void)num_sms;
  if (a.batch == 0) return cudaSuccess;
  dim3 block(32, kTpRows);
  dim3 grid((a.mult + 31) / 32, tp_chunks(a.batch));
  tp_fwd_kernel<PS><<<grid, block, 0, stream>>>(a);
  return cudaGetLastError();
}

template <int LI, int LS, int LO>
cudaError_t launch_tp_bwd(const TPArgs& a, int num_sms, cudaStream_t stream) {
  using PS = PathSet<LI, LS, LO>;
  (void)num_sms;
  const int chunks = tp_chunks(a.batch);
  if (a.batch > 0) {
    dim3 block(32, kTpRows);
    dim3 grid((a.mult + 31) / 32, chunks);
    tp_bwd_kernel<PS><<<grid, block, 0, stream>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (a.grad_w != nullptr) {
    const int n = PS::NP * a.mult;
    if (a.batch == 0) return cudaMemsetAsync(a.grad_w, 0, sizeof(float) * n, stream);
    tp_reduce_partials_kernel<<<(n + 255) / 256, 256, 0, stream>>>(chunks, n, a.partial, a.grad_w);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

// One translation unit per shape (the build passes CGTP_CFG_LI/LS/LO).
template cudaError_t launch_tp_fwd<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(const TPArgs&, int, cudaStream_t);
template cudaError_t launch_tp_bwd<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(const TPArgs&, int, cudaStream_t);

}  // namespace cgtp
