// CGTP convolution backward, node-centric over sources (CSC), for sm_100a.
//
// For edge e = (j -> i) with T_e^p[m1][m3] = sum_m2 C^p[m1,m2,m3] Y_e[l2,m2]:
//   t_p[m3][u]      = sum_m1 T_e^p[m1][m3] x[j][l1,m1][u]
//   grad_W[e][p][u] = sum_m3 g[i][l3,m3][u] t_p[m3][u]
//   s_p[m3][u]      = W_e[p][u] g[i][l3,m3][u]
//   grad_x[j][l1,m1][u] += sum_m3 T_e^p[m1][m3] s_p[m3][u]
//   grad_Y[e][l2,m2] = sum_p sum_{m1,m3} C^p[m1,m2,m3] sum_u x[j][l1,m1][u] s_p[m3][u]
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
#include "common.cuh"

namespace cgtp {
CGTP_DEFINE_CONSTANT_TABLES()
}  // namespace cgtp

#include "sh.cuh"

namespace cgtp {

namespace {

constexpr int kBwdThreads = 128;

template <int VEC>
struct VecIO;
template <>
struct VecIO<4> {
  static __device__ __forceinline__ void ld(float (&a)[4], const float* p) { f4_to(a, __ldg(reinterpret_cast<const float4*>(p))); }
  static __device__ __forceinline__ void ld_stream(float (&a)[4], const float* p) { f4_to(a, __ldcs(reinterpret_cast<const float4*>(p))); }
  static __device__ __forceinline__ void st(float* p, const float (&a)[4]) { *reinterpret_cast<float4*>(p) = to_f4(a); }
  static __device__ __forceinline__ void st_stream(float* p, const float (&a)[4]) { __stcs(reinterpret_cast<float4*>(p), to_f4(a)); }
};
template <>
struct VecIO<2> {
  static __device__ __forceinline__ void ld(float (&a)[2], const float* p) {
    const float2 v = __ldg(reinterpret_cast<const float2*>(p));
    a[0] = v.x; a[1] = v.y;
  }
  static __device__ __forceinline__ void ld_stream(float (&a)[2], const float* p) {
    const float2 v = __ldcs(reinterpret_cast<const float2*>(p));
    a[0] = v.x; a[1] = v.y;
  }
  static __device__ __forceinline__ void st(float* p, const float (&a)[2]) { *reinterpret_cast<float2*>(p) = make_float2(a[0], a[1]); }
  static __device__ __forceinline__ void st_stream(float* p, const float (&a)[2]) { __stcs(reinterpret_cast<float2*>(p), make_float2(a[0], a[1])); }
};

template <class PS>
__device__ __forceinline__ void compute_T_bwd(const float (&Y)[PS::NS], float* __restrict__ T) {
  static_for<0, PS::NP>([&](auto Pc) {
    constexpr int P = decltype(Pc)::value;
    constexpr int l1 = PS::D.l1[P], l2 = PS::D.l2[P], l3 = PS::D.l3[P];
    static_for<0, 2 * l3 + 1>([&](auto M3c) {
      constexpr int m3 = decltype(M3c)::value - l3;
      static_for<0, 2 * l1 + 1>([&](auto M1c) {
        constexpr int m1 = decltype(M1c)::value - l1;
        constexpr int ti = PS::t_index(P, m1, m3);
        if constexpr (ti >= 0) {
          float v = 0.f;
          static_for<0, 2 * l2 + 1>([&](auto M2c) {
            constexpr int m2 = decltype(M2c)::value - l2;
            if constexpr (cg_allowed(l1, l2, l3, m1, m2, m3)) {
              v = fmaf(c_cg[table_index(l1, l2, l3, m1, m2, m3)], Y[l2 * l2 + l2 + m2], v);
            }
          });
          T[ti] = v;
        }
      });
    });
    static_for<PS::D.tbase[P] + PS::D.tcount[P], PS::D.tbase[P + 1]>([&](auto Kc) {
      T[decltype(Kc)::value] = 0.f;
    });
  });
}

template <class PS>
constexpr bool first_of_l2(int k) {
  return k == 0 || PS::D.l2[PS::D.by_l2[k - 1]] != PS::D.l2[PS::D.by_l2[k]];
}

// One edge of the CSC row.  Paths are visited in (l2, l1, l3) order so that
// only one l2 block of the grad_Y partial is live at a time; each finished
// block goes to this lane's row of the shared reduction buffer (gyrow).  Each
// T entry is loaded once (four at a time) and used for t, grad_x and grad_Y.
template <class PS, int VEC, bool NEED_GY>
__device__ __forceinline__ void bwd_edge(const float* __restrict__ T, const float (&xr)[PS::NI][VEC],
                                         const float (&gr)[PS::NO][VEC], const float* __restrict__ wrow,
                                         float* __restrict__ gwrow, int mult, float (&gx)[PS::NI][VEC],
                                         float* __restrict__ gyrow) {
  float gy[PS::NS];
  static_for<0, PS::NP>([&](auto Kc) {
    constexpr int K = decltype(Kc)::value;
    constexpr int P = PS::D.by_l2[K];
    constexpr int l1 = PS::D.l1[P], l2 = PS::D.l2[P], l3 = PS::D.l3[P];
    constexpr int tb = PS::D.tbase[P], tc = PS::D.tcount[P];
    if constexpr (NEED_GY && first_of_l2<PS>(K)) {
#pragma unroll
      for (int m2 = 0; m2 < 2 * l2 + 1; ++m2) gy[l2 * l2 + m2] = 0.f;
    }
    float wv[VEC];
    VecIO<VEC>::ld_stream(wv, wrow + P * mult);
    float s[2 * l3 + 1][VEC], t[2 * l3 + 1][VEC];
#pragma unroll
    for (int m3 = 0; m3 < 2 * l3 + 1; ++m3)
#pragma unroll
      for (int c = 0; c < VEC; ++c) {
        s[m3][c] = wv[c] * gr[l3 * l3 + m3][c];
        t[m3][c] = 0.f;
      }
    static_for<0, (tc + 3) / 4>([&](auto Qc) {
      constexpr int q = decltype(Qc)::value;
      const float4 v4 = *reinterpret_cast<const float4*>(T + tb + 4 * q);
      const float tv4[4] = {v4.x, v4.y, v4.z, v4.w};
      static_for<0, 4>([&](auto Rc) {
        constexpr int k = 4 * q + decltype(Rc)::value;
        if constexpr (k < tc) {
          constexpr int m1 = PS::t_entry_m1(P, k), m3 = PS::t_entry_m3(P, k);
          constexpr int r1 = l1 * l1 + l1 + m1;
          const float tv = tv4[decltype(Rc)::value];
#pragma unroll
          for (int c = 0; c < VEC; ++c) {
            t[m3 + l3][c] = fmaf(tv, xr[r1][c], t[m3 + l3][c]);
            gx[r1][c] = fmaf(tv, s[m3 + l3][c], gx[r1][c]);
          }
          if constexpr (NEED_GY) {
            float av = 0.f;
#pragma unroll
            for (int c = 0; c < VEC; ++c) av = fmaf(xr[r1][c], s[m3 + l3][c], av);
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
    if (gwrow != nullptr) {
      float gw[VEC];
#pragma unroll
      for (int c = 0; c < VEC; ++c) {
        gw[c] = 0.f;
#pragma unroll
        for (int m3 = 0; m3 < 2 * l3 + 1; ++m3) gw[c] = fmaf(gr[l3 * l3 + m3][c], t[m3][c], gw[c]);
      }
      VecIO<VEC>::st_stream(gwrow + P * mult, gw);
    }
    if constexpr (NEED_GY && PS::D.last_of_l2[K]) {
#pragma unroll
      for (int m2 = 0; m2 < 2 * l2 + 1; ++m2) gyrow[l2 * l2 + m2] = gy[l2 * l2 + m2];
    }
  });
}

template <class PS, int VEC, bool NEED_GY>
__global__ void __launch_bounds__(kBwdThreads)
conv_bwd_kernel(ConvBwdArgs a, int lg_G, int S, int BT, int tstride) {
  constexpr int NI = PS::NI, NO = PS::NO, NS = PS::NS;
  constexpr int NSP = NS | 1;  // odd row stride: conflict-free transposed reduction
  extern __shared__ float4 smem_f4[];
  float* smem = reinterpret_cast<float*>(smem_f4);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int G = 1 << lg_G, gpw = 32 >> lg_G;
  const int grp = lane >> lg_G, gl = lane & (G - 1);
  const int group_floats = BT * tstride + 2 * ((BT + 3) & ~3);
  float* Tg = smem + (warp * gpw + grp) * group_floats;
  int* Eg = reinterpret_cast<int*>(Tg + BT * tstride);
  int* Ig = Eg + ((BT + 3) & ~3);
  // per warp: 32 x NSP floats for the grad_Y reduction
  float* red = smem + (kBwdThreads / 32) * gpw * group_floats + warp * 32 * NSP;

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
    float xr[NI][VEC], gx[NI][VEC];
#pragma unroll
    for (int r = 0; r < NI; ++r) {
      if (active) VecIO<VEC>::ld(xr[r], a.x + (node * NI + r) * a.mult + c0);
      else {
#pragma unroll
        for (int c = 0; c < VEC; ++c) xr[r][c] = 0.f;
      }
#pragma unroll
      for (int c = 0; c < VEC; ++c) gx[r][c] = 0.f;
    }

    for (int b0 = 0; b0 < maxdeg; b0 += BT) {
      for (int k = gl; k < BT; k += G) {
        const int kk = k0 + b0 + k;
        if (active && kk < k1) {
          const int e = __ldg(a.csc_edge + kk);
          float Y[NS];
          sh_of_vec<PS::LS>(__ldg(a.edge_vec + 3 * (long long)e), __ldg(a.edge_vec + 3 * (long long)e + 1),
                            __ldg(a.edge_vec + 3 * (long long)e + 2), Y);
          compute_T_bwd<PS>(Y, Tg + k * tstride);
          Eg[k] = e;
          Ig[k] = __ldg(a.csc_dst + kk);
        }
      }
      __syncwarp();
      const int nb = min(BT, maxdeg - b0);
      for (int k = 0; k < nb; ++k) {
        const bool valid = active && (k0 + b0 + k) < k1;
        float* rg = red + (grp * G) * NSP;  // this group's rows of the reduction buffer
        if constexpr (NEED_GY) {
#pragma unroll
          for (int b = 0; b < NS; ++b) rg[gl * NSP + b] = 0.f;  // l2 blocks no path touches
        }
        int e = 0;
        if (valid) {
          e = Eg[k];
          const long long i = Ig[k];
          float gr[NO][VEC];
#pragma unroll
          for (int r = 0; r < NO; ++r) VecIO<VEC>::ld(gr[r], a.grad_out + (i * NO + r) * a.mult + c0);
          const long long woff = (long long)e * PS::NP * a.mult + c0;
          bwd_edge<PS, VEC, NEED_GY>(Tg + k * tstride, xr, gr, a.w + woff,
                                     a.grad_w ? a.grad_w + woff : nullptr, a.mult, gx, rg + gl * NSP);
        }
        if constexpr (NEED_GY) {
          __syncwarp();
          if (valid) {
            float* dst = a.grad_sh + ((long long)slice * a.n_edges + e) * NS;
            for (int b = gl; b < NS; b += G) {
              float v = 0.f;
              for (int r = 0; r < G; ++r) v += rg[r * NSP + b];
              dst[b] = v;
            }
          }
          __syncwarp();
        }
      }
      __syncwarp();
    }
    if (active && a.grad_x != nullptr) {
#pragma unroll
      for (int r = 0; r < NI; ++r) VecIO<VEC>::st(a.grad_x + (node * NI + r) * a.mult + c0, gx[r]);
    }
  }
}

// grad_edge_vec[e] = (dY_e/dr_e)^T sum_s grad_sh[s][e]
template <int LS>
__global__ void sh_backward_kernel(int n_edges, int S, const float* __restrict__ edge_vec,
                                   const float* __restrict__ grad_sh, float* __restrict__ grad_edge_vec) {
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
    grad_edge_vec[3 * e] = d0;
    grad_edge_vec[3 * e + 1] = d1;
    grad_edge_vec[3 * e + 2] = d2;
  }
}

}  // namespace

template <class PS>
constexpr int bwd_vec() {
  return (PS::NI + PS::NO > 20) ? 2 : 4;
}

template <int LI, int LS, int LO>
int conv_bwd_slices(int mult) {
  using PS = PathSet<LI, LS, LO>;
  constexpr int VEC = bwd_vec<PS>();
  const int lanes = mult / VEC;
  int G = 1;
  while (G < 32 && lanes % (2 * G) == 0) G *= 2;
  return lanes / G;
}

template <int LI, int LS, int LO>
cudaError_t launch_conv_bwd(const ConvBwdArgs& a, int num_sms, cudaStream_t stream) {
  using PS = PathSet<LI, LS, LO>;
  constexpr int VEC = bwd_vec<PS>();
  constexpr int NSP = PS::NS | 1;
  const int lanes = a.mult / VEC;
  int G = 1;
  while (G < 32 && lanes % (2 * G) == 0) G *= 2;
  int lg_G = 0;
  while ((1 << lg_G) < G) ++lg_G;
  const int S = lanes / G;
  const int gpw = 32 / G;
  const int tstride = PS::NT > 0 ? PS::NT : 4;
  int BT = 4096 / (gpw * tstride);
  BT = BT < 1 ? 1 : (BT > 32 ? 32 : BT);
  const int group_floats = BT * tstride + 2 * ((BT + 3) & ~3);
  const bool need_gy = a.grad_edge_vec != nullptr;
  const size_t smem = sizeof(float) * ((size_t)group_floats * gpw * (kBwdThreads / 32) +
                                       (need_gy ? (size_t)(kBwdThreads / 32) * 32 * NSP : 0));
  const long long items = (long long)a.n_nodes * S;
  const long long groups_per_block = (long long)gpw * (kBwdThreads / 32);
  long long blocks = (items + groups_per_block - 1) / groups_per_block;
  cudaError_t err;
  auto run = [&](auto kern) -> cudaError_t {
    cudaError_t e2 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e2 != cudaSuccess) return e2;
    int per_sm = 0;
    e2 = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kBwdThreads, smem);
    if (e2 != cudaSuccess) return e2;
    if (per_sm < 1) per_sm = 1;
    const long long cap = (long long)num_sms * per_sm;
    long long nb = blocks > cap ? cap : blocks;
    if (nb < 1) nb = 1;
    kern<<<(unsigned)nb, kBwdThreads, smem, stream>>>(a, lg_G, S, BT, tstride);
    return cudaGetLastError();
  };
  if (need_gy) err = run(conv_bwd_kernel<PS, VEC, true>);
  else err = run(conv_bwd_kernel<PS, VEC, false>);
  if (err != cudaSuccess || !need_gy || a.n_edges == 0) return err;
  const int threads = 256;
  long long nbk = (a.n_edges + threads - 1) / threads;
  if (nbk > (long long)num_sms * 16) nbk = (long long)num_sms * 16;
  sh_backward_kernel<LS><<<(unsigned)nbk, threads, 0, stream>>>(a.n_edges, S, a.edge_vec, a.grad_sh,
                                                                 a.grad_edge_vec);
  return cudaGetLastError();
}

// One translation unit per shape (the build passes CGTP_CFG_LI/LS/LO).
template cudaError_t launch_conv_bwd<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(const ConvBwdArgs&, int,
                                                                         cudaStream_t);
template int conv_bwd_slices<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(int);

}  // namespace cgtp
