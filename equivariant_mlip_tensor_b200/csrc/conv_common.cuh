// Shared pieces of the node-centric convolution kernels: path groups, the
// per-edge T matrices of a group, vector loads/stores and per-lane
// asynchronous copies into shared memory.
//
// Include after CGTP_DEFINE_CONSTANT_TABLES (uses c_cg).
#pragma once

namespace cgtp {

// ---- vector I/O of VEC consecutive channels ----
template <int VEC>
struct VecIO;
template <>
struct VecIO<4> {
  static __device__ __forceinline__ void ld(float (&a)[4], const float* p) { f4_to(a, __ldg(reinterpret_cast<const float4*>(p))); }
  static __device__ __forceinline__ void lds(float (&a)[4], const float* p) { f4_to(a, *reinterpret_cast<const float4*>(p)); }
  static __device__ __forceinline__ void st(float* p, const float (&a)[4]) { *reinterpret_cast<float4*>(p) = to_f4(a); }
  static __device__ __forceinline__ void st_stream(float* p, const float (&a)[4]) { __stcs(reinterpret_cast<float4*>(p), to_f4(a)); }
  // asynchronous global -> shared copy of this lane's 16 bytes (L2 only)
  static __device__ __forceinline__ void cp_async(float* s, const float* g) {
    const unsigned sa = (unsigned)__cvta_generic_to_shared(s);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(g) : "memory");
  }
  // the same with an L2 eviction policy (streamed data: evict first)
  static __device__ __forceinline__ void cp_async_hint(float* s, const float* g, uint64_t pol) {
    const unsigned sa = (unsigned)__cvta_generic_to_shared(s);
    asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(sa), "l"(g), "l"(pol)
                 : "memory");
  }
};
template <>
struct VecIO<2> {
  static __device__ __forceinline__ void ld(float (&a)[2], const float* p) {
    const float2 v = __ldg(reinterpret_cast<const float2*>(p));
    a[0] = v.x; a[1] = v.y;
  }
  static __device__ __forceinline__ void lds(float (&a)[2], const float* p) {
    const float2 v = *reinterpret_cast<const float2*>(p);
    a[0] = v.x; a[1] = v.y;
  }
  static __device__ __forceinline__ void st(float* p, const float (&a)[2]) { *reinterpret_cast<float2*>(p) = make_float2(a[0], a[1]); }
  static __device__ __forceinline__ void st_stream(float* p, const float (&a)[2]) { __stcs(reinterpret_cast<float2*>(p), make_float2(a[0], a[1])); }
  static __device__ __forceinline__ void cp_async(float* s, const float* g) {
    const unsigned sa = (unsigned)__cvta_generic_to_shared(s);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(sa), "l"(g) : "memory");
  }
  static __device__ __forceinline__ void cp_async_hint(float* s, const float* g, uint64_t pol) {
    const unsigned sa = (unsigned)__cvta_generic_to_shared(s);
    asm volatile("cp.async.ca.shared.global.L2::cache_hint [%0], [%1], 8, %2;" ::"r"(sa), "l"(g), "l"(pol)
                 : "memory");
  }
};

// Weight rows are streamed (each read once per pass).  With
// CGTP_W_EVICT_FIRST their copies carry an L2 evict-first policy, so that
// they do not push the gathered feature and output-gradient rows (read once
// per edge, many times per pass) out of L2.
#ifndef CGTP_W_EVICT_FIRST
#define CGTP_W_EVICT_FIRST 0
#endif
__device__ __forceinline__ uint64_t stream_policy() {
  uint64_t pol = 0;
  if (CGTP_W_EVICT_FIRST) asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
template <int VEC>
__device__ __forceinline__ void cp_async_w(float* s, const float* g, uint64_t pol) {
  if constexpr (CGTP_W_EVICT_FIRST != 0) VecIO<VEC>::cp_async_hint(s, g, pol);
  else VecIO<VEC>::cp_async(s, g);
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// ---- path groups ----
// The convolution kernels split the paths into groups that share one l
// value: the backward groups by l1 (each group owns a block of grad_x rows),
// the forward by l3 (each group owns a block of output rows).  One launch
// per group keeps the per-thread state and the unrolled code small.
enum GroupKind { kByL1 = 0, kByL3 = 1, kAll = 2 };

template <class PS, int KIND, int V>
struct Grp {
  struct Data {
    int n;                       // paths in the group
    int path[kMaxPaths];         // path numbers, sorted by (l2, lexicographic)
    int lt[kMaxPaths + 1];       // group-local padded T offset of the k-th path
    bool first_l2[kMaxPaths];    // k-th path is the group's first with its l2
    bool last_l2[kMaxPaths];     // k-th path is the group's last with its l2
    int rlo, rhi;                // rows [rlo, rhi) of the gathered node tensor
  };
  static constexpr Data make() {
    Data d{};
    int lo = 99, hi = -1;
    for (int b = 0; b <= PS::LS; ++b)
      for (int p = 0; p < PS::D.np; ++p) {
        if (PS::D.l2[p] != b) continue;
        if (KIND != kAll && (KIND == kByL1 ? PS::D.l1[p] : PS::D.l3[p]) != V) continue;
        d.path[d.n++] = p;
        const int lo_other = KIND == kByL1 ? PS::D.l3[p] : PS::D.l1[p];
        lo = lo_other < lo ? lo_other : lo;
        hi = lo_other > hi ? lo_other : hi;
      }
    d.lt[0] = 0;
    for (int k = 0; k < d.n; ++k) {
      d.lt[k + 1] = d.lt[k] + (PS::D.tcount[d.path[k]] + 3) / 4 * 4;
      d.first_l2[k] = k == 0 || PS::D.l2[d.path[k - 1]] != PS::D.l2[d.path[k]];
      d.last_l2[k] = k + 1 == d.n || PS::D.l2[d.path[k + 1]] != PS::D.l2[d.path[k]];
    }
    d.rlo = d.n ? lo * lo : 0;
    d.rhi = d.n ? (hi + 1) * (hi + 1) : 0;
    return d;
  }
  static constexpr Data D = make();
  static constexpr int NP = D.n;
  static constexpr int NT = D.lt[D.n] > 0 ? D.lt[D.n] : 4;  // T floats per edge
  static constexpr int NROW = D.rhi - D.rlo;              // gathered node rows
  // rows of the group's own block (all output rows for kAll)
  static constexpr int NOWN = KIND == kAll ? PS::NO : 2 * V + 1;
  static constexpr int OWN0 = KIND == kAll ? 0 : V * V;    // first own row
  static constexpr bool FIRST = true;                      // initialises its rows
  static constexpr bool PERPATH = false;  // paths of one l3 summed into one block of rows
  static constexpr int NPK = 0, PL0 = 0;  // per-path layout only (see PathRowsGrp)
};

// T^p[m1][m3] = sum_m2 C^p[m1,m2,m3] Y[l2,m2] for the group's paths, packed
// per path in (m3, m1) order, each path padded to a multiple of 4 floats.
template <class PS, class GR>
__device__ __forceinline__ void compute_T_grp(const float (&Y)[PS::NS], float* __restrict__ T) {
  static_for<0, GR::NP>([&](auto Kc) {
    constexpr int K = decltype(Kc)::value;
    constexpr int P = GR::D.path[K];
    constexpr int l1 = PS::D.l1[P], l2 = PS::D.l2[P], l3 = PS::D.l3[P];
    constexpr int tc = PS::D.tcount[P], base = GR::D.lt[K];
    static_for<0, tc>([&](auto Ec) {
      constexpr int k = decltype(Ec)::value;
      constexpr int m1 = PS::t_entry_m1(P, k), m3 = PS::t_entry_m3(P, k);
      float v = 0.f;
      static_for<0, 2 * l2 + 1>([&](auto M2c) {
        constexpr int m2 = decltype(M2c)::value - l2;
        if constexpr (cg_allowed(l1, l2, l3, m1, m2, m3)) {
          v = fmaf(c_cg[table_index(l1, l2, l3, m1, m2, m3)], Y[l2 * l2 + l2 + m2], v);
        }
      });
      T[base + k] = v;
    });
    static_for<base + tc, GR::D.lt[K + 1]>([&](auto Zc) { T[decltype(Zc)::value] = 0.f; });
  });
}

// ---- per-path messages (the fully connected convolution) ----
// The messages of each path are kept apart in blocks by l3: block l3 holds
// [node][m3][rank][u] for the paths of that l3 in (l2, path number) order
// (the order in which the chunk planner visits them), and the blocks follow
// one another in increasing l3.
template <class PS>
constexpr int l3_rank(int p) {  // place of path p among the paths of its l3 block
  int r = 0;
  for (int q = 0; q < PS::D.np; ++q)
    if (PS::D.l3[q] == PS::D.l3[p] && (PS::D.l2[q] < PS::D.l2[p] || (PS::D.l2[q] == PS::D.l2[p] && q < p))) ++r;
  return r;
}
template <class PS>
constexpr int l3_count(int l3) {
  int n = 0;
  for (int q = 0; q < PS::D.np; ++q) n += PS::D.l3[q] == l3;
  return n;
}
// rows per node (paths x (2 l3 + 1)) of the blocks before block l3
template <class PS>
constexpr int l3_prefix_rows(int l3) {
  int r = 0;
  for (int l = 0; l < l3; ++l) r += l3_count<PS>(l) * (2 * l + 1);
  return r;
}

// ---- chunks: the launches of a kernel family ----
// Paths sorted by (key, l2, lexicographic), key = l1 (backward) or l3
// (forward), are cut into runs with one key value whose unrolled code per
// edge stays below a budget: a loop body much larger than about 20 KB of
// instructions stops fitting the instruction cache and the warps stall on
// instruction fetch.  Every run is one launch; the first run of a key
// initialises that key's block of rows, later runs add to it.  With merge,
// a run that holds a whole key may go on with the next keys while every one
// of them fits whole within the budget: the launch then owns the rows of
// keys key..key_hi (a small block, such as l1 = 0, rides along with the
// next instead of costing a pass of its own).
struct ChunkPlan {
  int n;                        // chunks
  int key[kMaxPaths];           // key value (l1 or l3) of chunk c (the first, when several)
  int key_hi[kMaxPaths];        // last key of chunk c
  int first[kMaxPaths];         // chunk c is order[first[c] .. first[c] + count[c])
  int count[kMaxPaths];
  bool first_of_key[kMaxPaths];
  int chain[kMaxPaths];         // chunks that continue a key's rows follow their predecessor: one chain each
  int order[kMaxPaths];         // paths sorted by (key, l2, lexicographic)
};

// Estimated unrolled instructions per edge and lane for one path.
template <class PS>
constexpr int path_cost(int p, int kind, int vec, bool gy) {
  const int tc = PS::D.tcount[p], n1 = 2 * PS::D.l1[p] + 1, n3 = 2 * PS::D.l3[p] + 1;
  if (kind == kByL3) return tc * vec + (tc + 3) / 4 + 1 + (n1 < n3 ? n1 : n3) * vec + 4;
  return tc * vec + (gy ? tc * vec + path_entries(PS::D.l1[p], PS::D.l2[p], PS::D.l3[p]) + n1 * vec : 0) +
         (tc + 3) / 4 + n3 + 2 * n1 * vec + 6;
}

// max_rows (forward by l3 only): at most this many output rows (sum of
// 2 l3 + 1 over the chunk's paths), for kernels that keep one block of
// accumulators per path.
template <class PS>
constexpr ChunkPlan make_chunk_plan(int kind, int vec, bool gy, int budget, int max_rows = 1 << 30,
                                   bool merge = false, bool merge_tail = false) {
  ChunkPlan c{};
  int k = 0;
  const int kmax = kind == kByL1 ? PS::LI : PS::LO;
  for (int key = 0; key <= kmax; ++key)
    for (int b = 0; b <= PS::LS; ++b)
      for (int p = 0; p < PS::D.np; ++p)
        if (PS::D.l2[p] == b && (kind == kByL1 ? PS::D.l1[p] : PS::D.l3[p]) == key) c.order[k++] = p;
  int start = 0;
  while (start < k) {
    const int key = kind == kByL1 ? PS::D.l1[c.order[start]] : PS::D.l3[c.order[start]];
    int end = start, cost = 0, rows = 0;
    while (end < k && (kind == kByL1 ? PS::D.l1[c.order[end]] : PS::D.l3[c.order[end]]) == key) {
      const int pc = path_cost<PS>(c.order[end], kind, vec, gy);
      const int pr = 2 * PS::D.l3[c.order[end]] + 1;
      if (end > start && (cost + pc > budget || rows + pr > max_rows)) break;
      cost += pc;
      rows += pr;
      ++end;
    }
    const bool whole = (start == 0 || (kind == kByL1 ? PS::D.l1[c.order[start - 1]] : PS::D.l3[c.order[start - 1]]) != key);
    int key_hi = key;
    if (merge && whole) {
      // append the following keys while each fits whole
      while (end < k) {
        const int nk = kind == kByL1 ? PS::D.l1[c.order[end]] : PS::D.l3[c.order[end]];
        int e2 = end, kc = 0, kr = 0;
        while (e2 < k && (kind == kByL1 ? PS::D.l1[c.order[e2]] : PS::D.l3[c.order[e2]]) == nk) {
          kc += path_cost<PS>(c.order[e2], kind, vec, gy);
          kr += 2 * PS::D.l3[c.order[e2]] + 1;
          ++e2;
        }
        if (cost + kc > budget || rows + kr > max_rows) {
          // merge_tail: the paths that would form the next key's last (small)
          // chunk, when they fit, start that key's rows here instead, and its
          // other chunks continue them
          if (merge_tail) {
            int ls = end, lc = 0, lr = 0;  // greedy chunks of key nk alone: the last one is [ls, e2)
            for (int q = end; q < e2; ++q) {
              const int pc = path_cost<PS>(c.order[q], kind, vec, gy);
              const int pr = 2 * PS::D.l3[c.order[q]] + 1;
              if (q > ls && (lc + pc > budget || lr + pr > max_rows)) ls = q, lc = 0, lr = 0;
              lc += pc;
              lr += pr;
            }
            if (ls > end && cost + lc <= budget && rows + lr <= max_rows) {
              // move order[ls, e2) to order[end, ...): one contiguous chunk
              for (int q = ls; q < e2; ++q) {
                const int p = c.order[q];
                for (int r = q; r > end + (q - ls); --r) c.order[r] = c.order[r - 1];
                c.order[end + (q - ls)] = p;
              }
              end += e2 - ls;
              cost += lc;
              rows += lr;
              key_hi = nk;
            }
          }
          break;
        }
        cost += kc;
        rows += kr;
        end = e2;
        key_hi = nk;
      }
    }
    c.key[c.n] = key;
    c.key_hi[c.n] = key_hi;
    c.first[c.n] = start;
    c.count[c.n] = end - start;
    c.first_of_key[c.n] = c.n == 0 || c.key_hi[c.n - 1] != key;
    c.chain[c.n] = c.n == 0 ? 0 : c.chain[c.n - 1] + (c.first_of_key[c.n] ? 1 : 0);
    ++c.n;
    start = end;
  }
  return c;
}

template <class PS, int KIND, int VEC, bool GY, int BUDGET, int MAX_ROWS = (1 << 30), bool MERGE = false,
          bool MERGE_TAIL = false>
struct Plan {
  static constexpr ChunkPlan P = make_chunk_plan<PS>(KIND, VEC, GY, BUDGET, MAX_ROWS, MERGE, MERGE_TAIL);
  static constexpr int N = P.n;
  static constexpr int CHAINS = P.n ? P.chain[P.n - 1] + 1 : 0;
};

// The paths of chunk CH of plan PL, with the same interface as Grp.
template <class PS, class PL, int CH>
struct Chunk {
  using Data = typename Grp<PS, kAll, 0>::Data;
  static constexpr int KEY = PL::P.key[CH];
  static constexpr int KEY_HI = PL::P.key_hi[CH];
  static constexpr bool FIRST = PL::P.first_of_key[CH];
  static constexpr Data make(bool by_l1) {
    Data d{};
    int lo = 99, hi = -1;
    // the chunk's paths by l2 (stable): the backward keeps one l2 block of its
    // harmonic-gradient partial live at a time, so all paths of one l2 must be
    // adjacent, also when the chunk holds several keys (each key's run is
    // already in l2 order)
    for (int b = 0; b <= PS::LS; ++b)
      for (int k = 0; k < PL::P.count[CH]; ++k) {
        const int p = PL::P.order[PL::P.first[CH] + k];
        if (PS::D.l2[p] != b) continue;
        d.path[d.n++] = p;
        const int other = by_l1 ? PS::D.l3[p] : PS::D.l1[p];
        lo = other < lo ? other : lo;
        hi = other > hi ? other : hi;
      }
    d.lt[0] = 0;
    for (int k = 0; k < d.n; ++k) {
      d.lt[k + 1] = d.lt[k] + (PS::D.tcount[d.path[k]] + 3) / 4 * 4;
      d.first_l2[k] = k == 0 || PS::D.l2[d.path[k - 1]] != PS::D.l2[d.path[k]];
      d.last_l2[k] = k + 1 == d.n || PS::D.l2[d.path[k + 1]] != PS::D.l2[d.path[k]];
    }
    d.rlo = d.n ? lo * lo : 0;
    d.rhi = d.n ? (hi + 1) * (hi + 1) : 0;
    return d;
  }
};
template <class PS, class PL, int CH, int KIND>
struct ChunkGrp : Chunk<PS, PL, CH> {
  using Base = Chunk<PS, PL, CH>;
  static constexpr typename Base::Data D = Base::make(KIND == kByL1);
  static constexpr int NP = D.n;
  static constexpr int NT = D.lt[D.n] > 0 ? D.lt[D.n] : 4;
  static constexpr int NROW = D.rhi - D.rlo;
  // own rows: the blocks of keys KEY..KEY_HI
  static constexpr int NOWN = (Base::KEY_HI + 1) * (Base::KEY_HI + 1) - Base::KEY * Base::KEY;
  static constexpr int OWN0 = Base::KEY * Base::KEY;
  static constexpr bool PERPATH = false;
  static constexpr int NPK = 0, PL0 = 0;
};

// Checks a launch's dynamic shared memory against the device's per-block
// opt-in limit before the attribute is set (a request beyond it is refused
// here rather than by the launch).
// Dynamic shared memory a block may opt in to (bytes; the same for every
// B200 in the process), or 0 when the device cannot be queried.
inline size_t smem_limit() {
  static int limit = -1;
  if (limit < 0) {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
      return 0;
    limit = v;
  }
  return (size_t)limit;
}
inline cudaError_t check_smem(size_t smem) {
  const size_t limit = smem_limit();
  if (limit == 0) return cudaErrorInvalidDevice;
  return smem <= limit ? cudaSuccess : cudaErrorInvalidConfiguration;
}

// Blocks of `threads` threads that one SM holds at once with `smem` bytes of
// dynamic shared memory and `regs` registers per thread (the limits of the
// device, read once: shared memory per SM and reserved per block, registers
// per SM in per-warp units of 256, blocks per SM).
inline int resident_blocks_per_sm(size_t smem, int regs, int threads) {
  static int sm_smem = -1, reserved = 0, sm_regs = 0, max_blocks = 0;
  if (sm_smem < 0) {
    int dev = 0, a = 0, b = 0, c = 0, d = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&a, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&b, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&c, cudaDevAttrMaxRegistersPerMultiprocessor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d, cudaDevAttrMaxBlocksPerMultiprocessor, dev) != cudaSuccess)
      return 1;
    reserved = b, sm_regs = c, max_blocks = d;
    sm_smem = a;
  }
  const int warps = (threads + 31) / 32;
  const int warp_regs = ((regs * 32 + 255) / 256) * 256;
  int n = max_blocks;
  if (warp_regs > 0) n = std::min(n, sm_regs / (warps * warp_regs));
  n = std::min(n, (int)(sm_smem / (smem + reserved)));
  return n;
}

// Edges per batch: T matrices of BT edges per group of lanes, sized so that a
// group's shared memory stays near 24 KB.
inline int pick_batch_staged(int gpw, int t_floats, int staging_floats, int budget_floats = 6144, int max_bt = 16) {
  const int budget = budget_floats / gpw - staging_floats;
  int bt = budget / (t_floats + 3);
  if (bt > max_bt) bt = max_bt;
  return bt < 1 ? 1 : bt;
}
// the same with two pipeline stages of stage_floats
inline int pick_batch(int gpw, int t_floats, int stage_floats, int budget_floats = 6144, int max_bt = 16) {
  return pick_batch_staged(gpw, t_floats, 2 * stage_floats, budget_floats, max_bt);
}

// Row split (log2 of the groups of lanes that share one work item): with few
// items, a warp holds one item instead of 32 / G, its groups taking every
// Q-th edge of the row, until there are about 8 warps per SM.  With
// max_warps > 1 and still few warps, *lg_W (log2 of the warps of one block,
// which then all take the same items) doubles while the grid stays within
// about 4 waves of 8 warps per SM.
inline int row_split(long long items, int gpw, int num_sms, int max_warps = 1, int* lg_W = nullptr) {
  int lg_Q = 0;
  const long long target = 8LL * num_sms;
  while ((1 << (lg_Q + 1)) <= gpw && items * (1LL << lg_Q) / gpw < target) ++lg_Q;
  if (lg_W != nullptr) {
    *lg_W = 0;
    const long long warps = items * (1LL << lg_Q) / gpw;
    while ((2 << *lg_W) <= max_warps && warps * (2LL << *lg_W) <= 4 * target) ++*lg_W;
  }
  return lg_Q;
}

// log2 of the channel lanes per group and the channel slices of a
// compile-time multiplicity km at vec channels per lane (as lane_geometry).
constexpr int kmult_lg_G(int km, int vec) {
  int g = 1, lg = 0;
  while (g < 32 && (km / vec) % (2 * g) == 0) g *= 2, ++lg;
  return lg;
}
constexpr int kmult_S(int km, int vec) { return km / vec / (1 << kmult_lg_G(km, vec)); }
// Plain forward and backward kernels also specialised for multiplicity 64 (1)
// or only 128 (0).
#ifndef CGTP_KMULT64
#define CGTP_KMULT64 1
#endif
// A compile-time multiplicity of at least 32 lanes x vec channels fills the
// warp with one item: no split of its rows inside or across warps.
constexpr bool kmult_whole_warp(int km, int vec) { return km >= 32 * vec; }

// Channel lanes per group (G, a power of two <= 32) and channel slices S for
// mult channels at VEC channels per lane.
inline void lane_geometry(int mult, int vec, int& G, int& lg_G, int& S) {
  const int lanes = mult / vec;
  G = 1;
  while (G < 32 && lanes % (2 * G) == 0) G *= 2;
  lg_G = 0;
  while ((1 << lg_G) < G) ++lg_G;
  S = lanes / G;
}

}  // namespace cgtp
