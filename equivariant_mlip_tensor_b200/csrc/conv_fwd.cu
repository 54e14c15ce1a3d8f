// CGTP convolution forward, node-centric over CSR rows, for sm_100a.
//
//   out[i][l3,m3][u] = sum_{e in row i} sum_p W_e[p][u] sum_m1 T_e^p[m1][m3] x[j_e][l1,m1][u]
//   T_e^p[m1][m3]    = sum_m2 C^p[m1,m2,m3] Y_e[l2,m2]
//
// ("LunaTP: Enabling Efficient and Scalable Tensor Product for Equivariant
// MLIPs", abstract: node-centric execution, path-group parallelism and reuse;
// this kernel is our own design for the B200.)
//
// Mapping.  A group of G lanes (G a power of two <= 32) owns one (row, channel
// slice) work item; each lane owns 4 consecutive channels (float4).  The
// group walks its row's edges in batches of BT: first every lane computes the
// harmonics and the packed T matrices of one edge of the batch (channel
// independent, coefficients from constant memory, so a batch costs one pass
// of this code whatever its size) into shared memory; then all lanes sweep
// the batch, streaming W_e (the dominant HBM stream, read once with an
// evict-first hint), gathering x_j (L2 resident), and accumulating the
// output row in registers.  Each output element is written once; there are
// no atomics.  The loops over paths, m3 and m1 are unrolled at compile time
// over the structural nonzero pattern of the real CG coefficients, so every
// register index is static.
#include "common.cuh"

namespace cgtp {
CGTP_DEFINE_CONSTANT_TABLES()
}  // namespace cgtp

#include "sh.cuh"

namespace cgtp {

namespace {

constexpr int kFwdThreads = 128;

// T matrices of one edge from its harmonics (packed layout of PathSet).
template <class PS>
__device__ __forceinline__ void compute_T(const float (&Y)[PS::NS], float* __restrict__ T) {
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
              constexpr int ci = table_index(l1, l2, l3, m1, m2, m3);
              v = fmaf(c_cg[ci], Y[l2 * l2 + l2 + m2], v);
            }
          });
          T[ti] = v;
        }
      });
    });
    // zero the padding so that float4 reads of the block see finite values
    static_for<PS::D.tbase[P] + PS::D.tcount[P], PS::D.tbase[P + 1]>([&](auto Kc) {
      T[decltype(Kc)::value] = 0.f;
    });
  });
}

// One edge: acc[l3,m3][c] += sum_p W[p][c] sum_m1 T[p][m1][m3] x[l1,m1][c].
template <class PS>
__device__ __forceinline__ void fwd_edge(const float* __restrict__ T, const float (&xr)[PS::NI][4],
                                         const float* __restrict__ wrow, int mult,
                                         float (&acc)[PS::NO][4]) {
  static_for<0, PS::NP>([&](auto Pc) {
    constexpr int P = decltype(Pc)::value;
    constexpr int l1 = PS::D.l1[P], l3 = PS::D.l3[P];
    constexpr int tb = PS::D.tbase[P], tn = PS::D.tbase[P + 1] - PS::D.tbase[P];
    float wv[4];
    f4_to(wv, ld_stream(wrow + P * mult));
    float tl[tn > 0 ? tn : 4];
    static_for<0, tn / 4>([&](auto Qc) {
      constexpr int q = decltype(Qc)::value;
      const float4 v = *reinterpret_cast<const float4*>(T + tb + 4 * q);
      tl[4 * q + 0] = v.x;
      tl[4 * q + 1] = v.y;
      tl[4 * q + 2] = v.z;
      tl[4 * q + 3] = v.w;
    });
    static_for<0, 2 * l3 + 1>([&](auto M3c) {
      constexpr int m3 = decltype(M3c)::value - l3;
      float t[4] = {0.f, 0.f, 0.f, 0.f};
      static_for<0, 2 * l1 + 1>([&](auto M1c) {
        constexpr int m1 = decltype(M1c)::value - l1;
        constexpr int ti = PS::t_index(P, m1, m3);
        if constexpr (ti >= 0) {
#pragma unroll
          for (int c = 0; c < 4; ++c) t[c] = fmaf(tl[ti - tb], xr[l1 * l1 + l1 + m1][c], t[c]);
        }
      });
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[l3 * l3 + l3 + m3][c] = fmaf(wv[c], t[c], acc[l3 * l3 + l3 + m3][c]);
    });
  });
}

template <class PS>
__global__ void __launch_bounds__(kFwdThreads)
conv_fwd_kernel(ConvFwdArgs a, int lg_G, int S, int BT, int tstride) {
  constexpr int NI = PS::NI, NO = PS::NO, NS = PS::NS;
  extern __shared__ float4 smem_f4[];
  float* smem = reinterpret_cast<float*>(smem_f4);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int G = 1 << lg_G, gpw = 32 >> lg_G;
  const int grp = lane >> lg_G, gl = lane & (G - 1);
  // per group: BT rows of T (stride tstride floats, 16-byte aligned) + BT source ids
  const int group_floats = BT * tstride + ((BT + 3) & ~3);
  float* Tg = smem + (warp * gpw + grp) * group_floats;
  int* Jg = reinterpret_cast<int*>(Tg + BT * tstride);

  const long long n_items = (long long)a.n_nodes * S;
  const long long warps_total = (long long)gridDim.x * (kFwdThreads / 32);
  for (long long base = ((long long)blockIdx.x * (kFwdThreads / 32) + warp) * gpw; base < n_items;
       base += warps_total * gpw) {
    const long long item = base + grp;
    const bool active = item < n_items;
    const int node = active ? int(item / S) : 0;
    const int slice = active ? int(item % S) : 0;
    const int c0 = (slice * G + gl) * 4;
    int e0 = 0, e1 = 0;
    if (active) {
      e0 = __ldg(a.row_ptr + node);
      e1 = __ldg(a.row_ptr + node + 1);
    }
    const int maxdeg = __reduce_max_sync(0xffffffffu, e1 - e0);
    float acc[NO][4];
#pragma unroll
    for (int k = 0; k < NO; ++k) acc[k][0] = acc[k][1] = acc[k][2] = acc[k][3] = 0.f;

    for (int b0 = 0; b0 < maxdeg; b0 += BT) {
      for (int k = gl; k < BT; k += G) {
        const int e = e0 + b0 + k;
        if (active && e < e1) {
          float Y[NS];
          sh_of_vec<PS::LS>(__ldg(a.edge_vec + 3 * (long long)e), __ldg(a.edge_vec + 3 * (long long)e + 1),
                            __ldg(a.edge_vec + 3 * (long long)e + 2), Y);
          compute_T<PS>(Y, Tg + k * tstride);
          Jg[k] = __ldg(a.col + e);
        }
      }
      __syncwarp();
      const int nb = min(BT, maxdeg - b0);
      for (int k = 0; k < nb; ++k) {
        const int e = e0 + b0 + k;
        if (active && e < e1) {
          const long long j = Jg[k];
          float xr[NI][4];
#pragma unroll
          for (int r = 0; r < NI; ++r) f4_to(xr[r], ld_ro(a.x + (j * NI + r) * a.mult + c0));
          fwd_edge<PS>(Tg + k * tstride, xr, a.w + (long long)e * PS::NP * a.mult + c0, a.mult, acc);
        }
      }
      __syncwarp();
    }
    if (active) {
#pragma unroll
      for (int r = 0; r < NO; ++r) st_f4(a.out + ((long long)node * NO + r) * a.mult + c0, to_f4(acc[r]));
    }
  }
}

}  // namespace

template <int LI, int LS, int LO>
cudaError_t launch_conv_fwd(const ConvFwdArgs& a, int num_sms, cudaStream_t stream) {
  using PS = PathSet<LI, LS, LO>;
  const int lanes = a.mult / 4;
  int G = 1;
  while (G < 32 && lanes % (2 * G) == 0) G *= 2;
  int lg_G = 0;
  while ((1 << lg_G) < G) ++lg_G;
  const int S = lanes / G;
  const int gpw = 32 / G;
  const int tstride = PS::NT > 0 ? PS::NT : 4;
  // batch size: about 16 KB of T per warp, at least one edge per lane when possible
  int BT = 4096 / (gpw * tstride);
  BT = BT < 1 ? 1 : (BT > 32 ? 32 : BT);
  const int group_floats = BT * tstride + ((BT + 3) & ~3);
  const size_t smem = sizeof(float) * (size_t)group_floats * gpw * (kFwdThreads / 32);
  auto kern = conv_fwd_kernel<PS>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFwdThreads, smem);
  if (err != cudaSuccess) return err;
  if (per_sm < 1) per_sm = 1;
  const long long items = (long long)a.n_nodes * S;
  const long long groups_per_block = (long long)gpw * (kFwdThreads / 32);
  long long blocks = (items + groups_per_block - 1) / groups_per_block;
  const long long cap = (long long)num_sms * per_sm;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  kern<<<(unsigned)blocks, kFwdThreads, smem, stream>>>(a, lg_G, S, BT, tstride);
  return cudaGetLastError();
}

// One translation unit per shape (the build passes CGTP_CFG_LI/LS/LO).
template cudaError_t launch_conv_fwd<CGTP_CFG_LI, CGTP_CFG_LS, CGTP_CFG_LO>(const ConvFwdArgs&, int,
                                                                         cudaStream_t);

}  // namespace cgtp
