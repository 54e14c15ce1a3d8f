// Neighbour list (CSR by destination, CSC by source) for sm_100a.
//
// Pairs within the cutoff form directed edges j -> i for the node-centric
// convolution ("LunaTP ...", abstract: node-centric CGTP convolutions).
// Bit-exact predicate, evaluated in fp64 with every operation rounded
// separately (no contraction into fused multiply-adds):
//   d = p_j - p_i;  periodic: d = d - L * rint(d / L);
//   edge iff ((dx*dx + dy*dy) + dz*dz) < rc*rc and i != j.
// One warp per destination row scans the candidate sources of the row's
// graph in index order, so each row comes out sorted by source; a ballot
// and a population count give every lane its output slot.  Counting, a
// single-block scan and filling are three stream-ordered launches with no
// host synchronisation.
#include <cuda_runtime.h>

#include "common.cuh"

namespace cgtp {

struct GraphArgs {
  const float* pos;
  int n;
  double L;
  bool pbc;
  double rc2;
  const int* graph_ptr;
  int n_graphs;
  int* row_ptr;
  int* col;
  float* edge_vec;
  int* csc_ptr;
  int* csc_edge;
  int* csc_dst;
  int max_edges;
  int* n_edges;
};

static __device__ __forceinline__ bool is_edge(const GraphArgs& a, double pix, double piy, double piz, int j,
                                        double& dx, double& dy, double& dz) {
  dx = __dsub_rn((double)__ldg(a.pos + 3 * (long long)j), pix);
  dy = __dsub_rn((double)__ldg(a.pos + 3 * (long long)j + 1), piy);
  dz = __dsub_rn((double)__ldg(a.pos + 3 * (long long)j + 2), piz);
  if (a.pbc) {
    dx = __dsub_rn(dx, __dmul_rn(a.L, rint(__ddiv_rn(dx, a.L))));
    dy = __dsub_rn(dy, __dmul_rn(a.L, rint(__ddiv_rn(dy, a.L))));
    dz = __dsub_rn(dz, __dmul_rn(a.L, rint(__ddiv_rn(dz, a.L))));
  }
  const double r2 = __dadd_rn(__dadd_rn(__dmul_rn(dx, dx), __dmul_rn(dy, dy)), __dmul_rn(dz, dz));
  return r2 < a.rc2;
}

static __device__ __forceinline__ void candidate_range(const GraphArgs& a, int i, int& g0, int& g1) {
  g0 = 0;
  g1 = a.n;
  if (a.graph_ptr != nullptr) {
    int lo = 0, hi = a.n_graphs - 1;  // largest g with graph_ptr[g] <= i
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(a.graph_ptr + mid) <= i) lo = mid;
      else hi = mid - 1;
    }
    g0 = __ldg(a.graph_ptr + lo);
    g1 = __ldg(a.graph_ptr + lo + 1);
  }
}

static __global__ void graph_count_kernel(GraphArgs a) {
  const int lane = threadIdx.x & 31;
  const long long nw = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long i = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); i < a.n; i += nw) {
    int g0, g1;
    candidate_range(a, (int)i, g0, g1);
    const double pix = __ldg(a.pos + 3 * i), piy = __ldg(a.pos + 3 * i + 1), piz = __ldg(a.pos + 3 * i + 2);
    int cnt = 0;
    for (int j0 = g0; j0 < g1; j0 += 32) {
      const int j = j0 + lane;
      double dx, dy, dz;
      const bool ok = j < g1 && j != i && is_edge(a, pix, piy, piz, j, dx, dy, dz);
      cnt += __popc(__ballot_sync(0xffffffffu, ok));
    }
    if (lane == 0) a.row_ptr[i + 1] = cnt;
  }
}

// In place: v[1..n] counts -> inclusive prefix sums, v[0] = 0 (one block).
static __device__ void block_scan_counts(int* v, int n) {
  __shared__ int warp_sums[32];
  __shared__ int carry;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nwarps = blockDim.x >> 5;
  if (tid == 0) {
    carry = 0;
    v[0] = 0;
  }
  __syncthreads();
  for (int base = 0; base < n; base += blockDim.x) {
    const int k = base + tid;
    int x = k < n ? v[k + 1] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int s = lane < nwarps ? warp_sums[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      if (lane < nwarps) warp_sums[lane] = s;
    }
    __syncthreads();
    const int prefix = carry + (wid > 0 ? warp_sums[wid - 1] : 0);
    if (k < n) v[k + 1] = x + prefix;
    __syncthreads();
    if (tid == blockDim.x - 1) carry = prefix + x;
    __syncthreads();
  }
}

static __global__ void graph_scan_kernel(GraphArgs a) {
  block_scan_counts(a.row_ptr, a.n);
  __syncthreads();
  for (int k = threadIdx.x; k <= a.n; k += blockDim.x) a.csc_ptr[k] = a.row_ptr[k];
  if (threadIdx.x == 0) *a.n_edges = a.row_ptr[a.n];
}

static __global__ void graph_fill_kernel(GraphArgs a) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  const long long nw = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long i = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); i < a.n; i += nw) {
    int g0, g1;
    candidate_range(a, (int)i, g0, g1);
    const double pix = __ldg(a.pos + 3 * i), piy = __ldg(a.pos + 3 * i + 1), piz = __ldg(a.pos + 3 * i + 2);
    int base = a.row_ptr[i];
    for (int j0 = g0; j0 < g1; j0 += 32) {
      const int j = j0 + lane;
      double dx = 0.0, dy = 0.0, dz = 0.0;
      const bool ok = j < g1 && j != i && is_edge(a, pix, piy, piz, j, dx, dy, dz);
      const unsigned m = __ballot_sync(0xffffffffu, ok);
      const int pos = base + __popc(m & lt);
      if (ok && pos < a.max_edges) {
        a.col[pos] = j;
        a.edge_vec[3 * (long long)pos] = (float)dx;
        a.edge_vec[3 * (long long)pos + 1] = (float)dy;
        a.edge_vec[3 * (long long)pos + 2] = (float)dz;
      }
      base += __popc(m);
    }
  }
}

// CSC by source of a symmetric graph: the k-th neighbour i of j (CSR row j)
// is the destination of edge (j -> i), which sits in CSR row i where col == j.
static __global__ void graph_csc_kernel(GraphArgs a) {
  if (a.row_ptr[a.n] > a.max_edges) return;  // truncated graph: caller must rebuild
  const int lane = threadIdx.x & 31;
  const long long nw = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long j = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); j < a.n; j += nw) {
    const int k0 = a.row_ptr[j], k1 = a.row_ptr[j + 1];
    for (int k = k0 + lane; k < k1; k += 32) {
      const int i = a.col[k];
      int lo = a.row_ptr[i], hi = a.row_ptr[i + 1];  // lower_bound of j in col[lo..hi)
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (a.col[mid] < (int)j) lo = mid + 1;
        else hi = mid;
      }
      a.csc_edge[k] = lo;
      a.csc_dst[k] = i;
    }
  }
}

static int warp_grid(long long rows, int num_sms, int warps_per_block) {
  long long b = (rows + warps_per_block - 1) / warps_per_block;
  const long long cap = (long long)num_sms * 32;
  if (b > cap) b = cap;
  return (int)(b < 1 ? 1 : b);
}

cudaError_t launch_graph_build(const float* pos, int n, float box_len, float rc, const int* graph_ptr,
                               int n_graphs, int* row_ptr, int* col, float* edge_vec, int* csc_ptr,
                               int* csc_edge, int* csc_dst, int max_edges, int* n_edges, int num_sms,
                               cudaStream_t stream) {
  GraphArgs a;
  a.pos = pos;
  a.n = n;
  a.pbc = box_len > 0.f;
  a.L = (double)box_len;
  const double rc64 = (double)rc;
  a.rc2 = rc64 * rc64;
  a.graph_ptr = graph_ptr;
  a.n_graphs = n_graphs;
  a.row_ptr = row_ptr;
  a.col = col;
  a.edge_vec = edge_vec;
  a.csc_ptr = csc_ptr;
  a.csc_edge = csc_edge;
  a.csc_dst = csc_dst;
  a.max_edges = max_edges;
  a.n_edges = n_edges;
  const int wpb = 8;
  const int grid = warp_grid(n, num_sms, wpb);
  if (n > 0) {
    graph_count_kernel<<<grid, 32 * wpb, 0, stream>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  graph_scan_kernel<<<1, 1024, 0, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || n == 0) return e;
  graph_fill_kernel<<<grid, 32 * wpb, 0, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  graph_csc_kernel<<<grid, 32 * wpb, 0, stream>>>(a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- transpose
static __global__ void transpose_count_kernel(int n_edges, const int* __restrict__ col, int* __restrict__ cnt) {
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n_edges;
       e += (long long)gridDim.x * blockDim.x)
    atomicAdd(cnt + col[e] + 1, 1);
}

static __global__ void transpose_scan_kernel(int n, int* csc_ptr) { block_scan_counts(csc_ptr, n); }

static __global__ void transpose_fill_kernel(int n, const int* __restrict__ row_ptr, const int* __restrict__ col,
                                      const int* __restrict__ csc_ptr, int* __restrict__ cursor,
                                      int* __restrict__ csc_edge) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    for (int e = row_ptr[i]; e < row_ptr[i + 1]; ++e) {
      const int j = col[e];
      const int slot = atomicAdd(cursor + j, 1);
      csc_edge[csc_ptr[j] + slot] = e;
    }
}

// Each CSC row sorted by edge number, i.e. by (destination, source): the
// atomic slots above come in arbitrary order; this makes the result unique.
static __global__ void transpose_sort_kernel(int n, const int* __restrict__ row_ptr, const int* __restrict__ csc_ptr,
                                      int* __restrict__ csc_edge, int* __restrict__ csc_dst) {
  for (long long j = blockIdx.x * (long long)blockDim.x + threadIdx.x; j < n; j += (long long)gridDim.x * blockDim.x) {
    const int k0 = csc_ptr[j], k1 = csc_ptr[j + 1];
    for (int k = k0 + 1; k < k1; ++k) {
      const int v = csc_edge[k];
      int q = k - 1;
      while (q >= k0 && csc_edge[q] > v) {
        csc_edge[q + 1] = csc_edge[q];
        --q;
      }
      csc_edge[q + 1] = v;
    }
    for (int k = k0; k < k1; ++k) {
      const int e = csc_edge[k];
      int lo = 0, hi = n - 1;  // row of e: largest i with row_ptr[i] <= e
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (row_ptr[mid] <= e) lo = mid;
        else hi = mid - 1;
      }
      csc_dst[k] = lo;
    }
  }
}

cudaError_t launch_csr_transpose(int n, int n_edges, const int* row_ptr, const int* col, int* csc_ptr,
                                 int* csc_edge, int* csc_dst, int* ws, int num_sms, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(csc_ptr, 0, sizeof(int) * (n + 1), stream);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(ws, 0, sizeof(int) * n, stream);
  if (e != cudaSuccess) return e;
  const int tb = 256;
  long long g = ((long long)n_edges + tb - 1) / tb;
  if (g > num_sms * 8LL) g = num_sms * 8LL;
  if (n_edges > 0) {
    transpose_count_kernel<<<(int)(g < 1 ? 1 : g), tb, 0, stream>>>(n_edges, col, csc_ptr);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  transpose_scan_kernel<<<1, 1024, 0, stream>>>(n, csc_ptr);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (n == 0 || n_edges == 0) return cudaSuccess;
  long long gn = ((long long)n + tb - 1) / tb;
  if (gn > num_sms * 8LL) gn = num_sms * 8LL;
  transpose_fill_kernel<<<(int)gn, tb, 0, stream>>>(n, row_ptr, col, csc_ptr, ws, csc_edge);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  transpose_sort_kernel<<<(int)gn, tb, 0, stream>>>(n, row_ptr, csc_ptr, csc_edge, csc_dst);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- validation
// Flag bits (OR-ed into *flags): 1 CSR offsets (row_ptr[0] != 0,
// row_ptr[n] != n_edges or decreasing), 2 CSR source out of range,
// 4 zero-length edge vector, 8 non-finite edge vector, 16 CSC offsets,
// 32 CSC edge number or destination out of range.  Any array may be null
// (not checked).
static __global__ void graph_validate_kernel(int n, int n_edges, const int* __restrict__ row_ptr,
                                             const int* __restrict__ col, const float* __restrict__ edge_vec,
                                             const int* __restrict__ csc_ptr, const int* __restrict__ csc_edge,
                                             const int* __restrict__ csc_dst, int* __restrict__ flags) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  const long long t0 = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  int f = 0;
  if (row_ptr != nullptr) {
    if (t0 == 0 && (row_ptr[0] != 0 || row_ptr[n] != n_edges)) f |= 1;
    for (long long i = t0; i < n; i += stride)
      if (row_ptr[i + 1] < row_ptr[i]) f |= 1;
  }
  if (csc_ptr != nullptr) {
    if (t0 == 0 && (csc_ptr[0] != 0 || csc_ptr[n] != n_edges)) f |= 16;
    for (long long i = t0; i < n; i += stride)
      if (csc_ptr[i + 1] < csc_ptr[i]) f |= 16;
  }
  for (long long e = t0; e < n_edges; e += stride) {
    if (col != nullptr) {
      const int j = col[e];
      if (j < 0 || j >= n) f |= 2;
    }
    if (csc_edge != nullptr) {
      const int k = csc_edge[e];
      if (k < 0 || k >= n_edges) f |= 32;
    }
    if (csc_dst != nullptr) {
      const int d = csc_dst[e];
      if (d < 0 || d >= n) f |= 32;
    }
    if (edge_vec != nullptr) {
      const float x = edge_vec[3 * e], y = edge_vec[3 * e + 1], z = edge_vec[3 * e + 2];
      if (!(isfinite(x) && isfinite(y) && isfinite(z))) f |= 8;
      else if (x == 0.f && y == 0.f && z == 0.f) f |= 4;
    }
  }
  if (f) atomicOr(flags, f);
}

cudaError_t launch_graph_validate(int n, int n_edges, const int* row_ptr, const int* col, const float* edge_vec,
                                  const int* csc_ptr, const int* csc_edge, const int* csc_dst, int* flags,
                                  int num_sms, cudaStream_t stream) {
  graph_validate_kernel<<<num_sms * 4, 256, 0, stream>>>(n, n_edges, row_ptr, col, edge_vec, csc_ptr, csc_edge,
                                                          csc_dst, flags);
  return cudaGetLastError();
}

cudaError_t launch_graph_check(int n, int n_edges, const int* row_ptr, const int* col, const float* edge_vec,
                               int* flags, int num_sms, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(flags, 0, sizeof(int), stream);
  if (e != cudaSuccess) return e;
  return launch_graph_validate(n, n_edges, row_ptr, col, edge_vec, nullptr, nullptr, nullptr, flags, num_sms,
                               stream);
}

}  // namespace cgtp
