/*
 * cgtp.h -- C ABI of the B200 (sm_100a) Clebsch-Gordan tensor-product
 * convolution library (libcgtp.so).
 *
 * The operation ("LunaTP: Enabling Efficient and Scalable Tensor Product for
 * Equivariant MLIPs", abstract: node-centric CGTP convolutions and their
 * derivatives; selection rules from "Tensor Decomposition Networks for
 * Accelerating Machine Learning Force Field Computations", reply to reviewer
 * S6y1).  For every directed edge e = (j -> i) with edge vector
 * r_e = pos_j - pos_i, real spherical harmonics Y_e = Y(r_e / |r_e|) and
 * weights W_e[p][u]:
 *
 *   out[i][l3,m3][u] = sum_{e in row i} sum_{p=(l1,l2,l3)} W_e[p][u]
 *                      sum_{m1,m2} C^p[m1,m2,m3] x[j][l1,m1][u] Y_e[l2,m2]
 *
 * over every path with l1 <= lmax_in, l2 <= lmax_sh and
 * |l1-l2| <= l3 <= min(l1+l2, lmax_out).  Paths are numbered in
 * lexicographic (l1, l2, l3) order.
 *
 * Conventions shared by every entry point
 *  - Layouts: irreps features are [node][l*l + m + l][u] with the channel u
 *    fastest (fp32); weights are [edge][path][u] (fp32); edge vectors are
 *    [edge][3] (fp32); the real basis orders the l = 1 block as (y, z, x);
 *    harmonics use component normalisation (sum_m Y_lm^2 = 2l + 1,
 *    Y_00 = 1); CG coefficients are the unitary real-basis ones.
 *  - Graphs: CSR by destination (row_ptr [N+1], col [E] = source of each
 *    edge, rows ascending, sources ascending within a row).  The CSC view by
 *    source (csc_ptr [N+1], csc_edge [E] = CSR edge number, csc_dst [E] =
 *    destination) lists each source's edges in ascending destination order.
 *    All indices are int32.
 *  - Pointers: "device" arguments are caller-owned device memory; the
 *    library never frees or retains them.  Feature, weight and output arrays
 *    must be 16-byte aligned (they are read and written as float4).
 *  - Streams: every call is asynchronous on the given cudaStream_t (passed
 *    as void*, NULL = legacy default stream); nothing synchronises unless
 *    stated.
 *  - Errors: every call returns a cgtp_status.  Invalid arguments are found
 *    on the host before any launch (CGTP_ERR_INVALID_ARG /
 *    CGTP_ERR_UNSUPPORTED) and nothing is launched.  A launch failure
 *    returns CGTP_ERR_CUDA; cgtp_last_cuda_error() gives the CUDA code.
 *    Nothing aborts, throws or exits across this boundary.
 *  - Zero-length edges (coincident atoms) have no direction: their
 *    harmonics are Y_00 = 1 and 0 for l > 0, with a zero derivative.
 */
#ifndef CGTP_H
#define CGTP_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CGTP_OK = 0,
  CGTP_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, negative size, ...  */
  CGTP_ERR_UNSUPPORTED = 2,  /* (lmax_in, lmax_sh, lmax_out, mult) not built  */
  CGTP_ERR_BAD_GRAPH = 3,    /* reported by cgtp_graph_check                   */
  CGTP_ERR_OOM = 4,          /* host allocation failed                          */
  CGTP_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed            */
  CGTP_ERR_TABLE = 6,        /* CG table construction failed its own checks    */
  CGTP_ERR_WORKSPACE = 7     /* workspace missing or smaller than required      */
} cgtp_status;

typedef struct cgtp_plan_s* cgtp_plan;

/* What a plan computes.  Every entry point states the modes it accepts and
 * returns CGTP_ERR_INVALID_ARG for a plan of another mode.
 *  CGTP_MODE_CONV_UVU         the channelwise convolution over a graph, one
 *                             weight per edge, path and channel (w [E][P][u]):
 *                             cgtp_conv_forward / _backward / _double_backward,
 *                             cgtp_radial_*;
 *  CGTP_MODE_PAIR_UVU         the edge-free channelwise product of batched pairs
 *                             and its CP-decomposed surrogate: cgtp_tp_*, cgtp_cp_*;
 *  CGTP_MODE_CONV_UVU_SHARED  the channelwise convolution with one weight row per
 *                             edge shared by every path (path stride 0, w [E][u];
 *                             "Tensor Decomposition Networks ...", reply to
 *                             reviewer oXft): cgtp_conv_forward / _backward,
 *                             cgtp_radial_*;
 *  CGTP_MODE_CONV_UVW         the fully connected convolution (channelwise
 *                             messages mixed across channels per path;
 *                             "Tensor Decomposition Networks ...", reply to
 *                             reviewer cmnz): cgtp_uvw_*, cgtp_radial_*. */
typedef enum {
  CGTP_MODE_CONV_UVU = 0,
  CGTP_MODE_PAIR_UVU = 1,
  CGTP_MODE_CONV_UVU_SHARED = 2,
  CGTP_MODE_CONV_UVW = 3
} cgtp_mode;

/* Human-readable name of a status code (static string). */
const char* cgtp_status_string(cgtp_status s);

/* CUDA error code (cudaError_t as int) of the last CGTP_ERR_CUDA on this
 * host thread, 0 if none. */
int cgtp_last_cuda_error(void);

/* ---------------------------------------------------------------------------
 * Plan: the path list and the real CG coefficients of one irreps shape, for
 * one mode.  ("Tensor Decomposition Networks ...", reply to S6y1: only
 * triples obeying |l1-l2| <= l3 <= l1+l2 and m3 = m1+m2 are nonzero.)
 * Builds the coefficients on the host (fp64, by the angular-momentum
 * lowering operator and the complex-to-real change of basis), checks them,
 * and uploads them once per device to constant memory (synchronous copy on
 * the current device).  mult must be a positive multiple of 4.
 * Returns CGTP_ERR_INVALID_ARG for a negative l, a bad mult or an unknown
 * mode, and CGTP_ERR_UNSUPPORTED for a shape whose kernels are not compiled
 * in for the mode (see cgtp_supported).  The plan owns its host path list
 * and, in checked mode, 16 bytes of device memory; nothing else.
 * ------------------------------------------------------------------------- */
cgtp_status cgtp_plan_create(int lmax_in, int lmax_sh, int lmax_out, int mult, cgtp_mode mode,
                             cgtp_plan* plan);
cgtp_status cgtp_plan_destroy(cgtp_plan plan);

/* 1 if the kernels of (lmax_in, lmax_sh, lmax_out) are compiled in for the
 * mode, else 0.  Compiled shapes, all with lmax_in, lmax_out <= 3 and
 * lmax_sh <= 4:
 *  CONV_UVU, PAIR_UVU: every interaction shape (lmax_in == lmax_out), every
 *    embedding shape (lmax_in == 0) and every read-out shape (lmax_out == 0);
 *  CONV_UVU_SHARED, CONV_UVW: (0,0,0), (1,1,1), (1,2,1), (2,2,2), (2,4,2),
 *    (3,3,3).
 * Host only. */
int cgtp_supported(int lmax_in, int lmax_sh, int lmax_out, cgtp_mode mode);

/* Checked mode (off by default).  With checked != 0, every convolution call
 * of the plan first validates, on the device and in its stream, the graph
 * arrays it is given, OR-ing the bits of cgtp_graph_check (plus 16 = CSC
 * offsets not monotone or not ending at n_edges, 32 = a CSC edge number or
 * destination out of range) into the plan's flags.  If an offset or index
 * bit (1, 2, 16 or 32) is set, the call's convolution kernels do no work
 * (their outputs are left unspecified), so an invalid graph cannot make them
 * read or write out of bounds.  The first switch-on allocates the flags
 * (16 bytes) on the current device; the plan's checked calls must then run
 * on that device (CGTP_ERR_CUDA otherwise). */
cgtp_status cgtp_plan_set_checked(cgtp_plan plan, int checked);

/* Reads and clears the flags that the plan's checked-mode calls recorded:
 * synchronises the device (every stream), stores the bits in *flags
 * (nullable) and returns CGTP_ERR_BAD_GRAPH if any bit is set, CGTP_OK if
 * none (also for a plan never put in checked mode).  Not for use during
 * stream capture. */
cgtp_status cgtp_plan_check(cgtp_plan plan, int* flags);

/* Number of paths; if paths_l1l2l3 is not NULL it receives 3*n_paths ints
 * (l1, l2, l3 per path, lexicographic).  n_cg_nonzero (nullable) receives
 * the number of nonzero real CG entries over all paths.  Host only. */
cgtp_status cgtp_plan_info(cgtp_plan plan, int* n_paths, int* paths_l1l2l3, int* n_cg_nonzero);

/* Host-only: the dense real-basis CG block of path (l1, l2, l3), all <= 4,
 * as (2l1+1)*(2l2+1)*(2l3+1) doubles in [m1][m2][m3] order, computed by the
 * same generator that feeds the kernels.  Needs no GPU. */
cgtp_status cgtp_cg_block(int l1, int l2, int l3, double* out);

/* ---------------------------------------------------------------------------
 * Neighbour list (CSR by destination + CSC by source), brute force over the
 * candidate pairs of each graph.  (The convolution sums over the neighbours
 * of each atom within a cutoff, as interatomic potentials do: "LunaTP ...",
 * abstract, convolutions over atomic neighbourhoods; the machine review of
 * "AccelNet", summary: sums over the neighbours within the cutoff.  The
 * pages fix no algorithm; this one is exact.)  Bit-exact contract:
 *   d = p_j - p_i per axis in fp64 (positions upcast from fp32);
 *   periodic box (side box_len > 0): d <- d - L*rint(d/L), each operation
 *   rounded separately (rint: halves to even); box_len <= 0 means no box;
 *   edge when ((dx*dx + dy*dy) + dz*dz) < rc*rc in fp64 without fused
 *   multiply-add, rc*rc formed in fp64 from the fp32 cutoff, i != j;
 *   edge_vec = (float)d.
 * pos: device [n][3].  graph_ptr: device [n_graphs+1] start offsets of
 * contiguous graphs (pairs only within a graph), or NULL for one graph.
 * Outputs (device): row_ptr [n+1], col [max_edges], edge_vec [max_edges][3],
 * csc_ptr [n+1], csc_edge [max_edges], csc_dst [max_edges], n_edges [1].
 * If the true edge count exceeds max_edges, *n_edges holds the true count,
 * row_ptr is complete, and only the edges below max_edges are written (the
 * caller must check *n_edges and rebuild with more room).  The CSC arrays
 * use the symmetry of the predicate (j in N(i) iff i in N(j)).
 * Requires rc < box_len/2 with a box.  No host synchronisation.
 * ------------------------------------------------------------------------- */
cgtp_status cgtp_graph_build(const float* pos, int n, float box_len, float rc,
                             const int* graph_ptr, int n_graphs,
                             int* row_ptr, int* col, float* edge_vec,
                             int* csc_ptr, int* csc_edge, int* csc_dst,
                             int max_edges, int* n_edges, void* stream);

/* CSC view of an arbitrary CSR graph (no symmetry assumed).
 * workspace: device, at least n*sizeof(int) bytes (zeroed by the call). */
cgtp_status cgtp_csr_transpose(int n, int n_edges, const int* row_ptr, const int* col,
                               int* csc_ptr, int* csc_edge, int* csc_dst,
                               void* workspace, size_t workspace_bytes, void* stream);

/* Device-side validation of a CSR graph (the checks that checked-mode plans
 * run; an addition of this library): sets bits of *flags (device int,
 * cleared by the call): 1 = row_ptr not monotone or row_ptr[0] != 0 or
 * row_ptr[n] != n_edges, 2 = col out of range, 4 = zero-length edge vector,
 * 8 = non-finite edge vector. */
cgtp_status cgtp_graph_check(int n, int n_edges, const int* row_ptr, const int* col,
                             const float* edge_vec, int* flags, void* stream);

/* ---------------------------------------------------------------------------
 * Real spherical harmonics of edge directions (materialised; the
 * convolution kernels compute them in registers).  Y: device
 * [n_edges][(lmax_sh+1)^2]; dY (nullable): device [n_edges][(lmax_sh+1)^2][3]
 * = dY/d(edge_vec).  lmax_sh <= 4.
 * ------------------------------------------------------------------------- */
cgtp_status cgtp_spherical_harmonics(int lmax_sh, int n_edges, const float* edge_vec,
                                     float* Y, float* dY, void* stream);

/* ---------------------------------------------------------------------------
 * Convolution forward (node-centric: one owner per destination row, no
 * atomics).  Modes CONV_UVU and CONV_UVU_SHARED.
 * x: [n_nodes][(lmax_in+1)^2][mult]; w: [n_edges][n_paths][mult], or
 * [n_edges][mult] (one row shared by every path) for CONV_UVU_SHARED;
 * out: [n_nodes][(lmax_out+1)^2][mult] (overwritten).
 * ------------------------------------------------------------------------- */
cgtp_status cgtp_conv_forward(cgtp_plan plan, int n_nodes, int n_edges,
                              const int* row_ptr, const int* col, const float* edge_vec,
                              const float* x, const float* w, float* out, void* stream);

/* Bytes of device workspace cgtp_conv_backward needs when grad_edge_vec is
 * requested (0 otherwise is also accepted).  Modes CONV_UVU,
 * CONV_UVU_SHARED, CONV_UVW. */
cgtp_status cgtp_conv_backward_workspace_size(cgtp_plan plan, int n_edges, size_t* bytes);

/* ---------------------------------------------------------------------------
 * Convolution backward, node-centric over sources (CSC), one read of W
 * (modes CONV_UVU and CONV_UVU_SHARED; with the latter w and grad_w are
 * [n_edges][mult] and grad_w[e] is the sum over paths of the per-path weight
 * gradients):
 *   grad_x[j] = sum_{e: src=j} sum_p W_e[p] (T_e^p)^T grad_out[dst(e)]
 *   grad_w[e][p][u] = sum C x[j] Y_e grad_out[i]
 *   grad_edge_vec[e] = (dY_e/dr_e)^T sum_u sum_p W x grad_out C
 * with T_e^p[m1][m3] = sum_m2 C^p[m1,m2,m3] Y_e[l2,m2].
 * grad_x, grad_w, grad_edge_vec are nullable (not computed when NULL) and
 * overwritten.  grad_edge_vec needs workspace of the size reported by
 * cgtp_conv_backward_workspace_size (device, 256-byte aligned).
 * Streams: the launches of different l1 blocks run on side streams of the
 * library, forked from `stream` with an event and joined back before the call
 * returns, so the call is ordered on `stream` like a single launch.  The first
 * call on a device creates those streams and events: make it before any
 * stream capture.
 * ------------------------------------------------------------------------- */
cgtp_status cgtp_conv_backward(cgtp_plan plan, int n_nodes, int n_edges,
                               const int* csc_ptr, const int* csc_edge, const int* csc_dst,
                               const float* edge_vec, const float* x, const float* w,
                               const float* grad_out, float* grad_x, float* grad_w,
                               float* grad_edge_vec, void* workspace, size_t workspace_bytes,
                               void* stream);

/* Bytes of device workspace cgtp_conv_double_backward needs when
 * gg_edge_vec or d_edge_vec is given.  Mode CONV_UVU. */
cgtp_status cgtp_conv_double_backward_workspace_size(cgtp_plan plan, int n_edges, size_t* bytes);

/* ---------------------------------------------------------------------------
 * Double backward: the adjoint of cgtp_conv_backward, the higher-order
 * derivative that force training needs ("LunaTP ...", abstract: derivative
 * computation).  Mode CONV_UVU.  With (grad_x, grad_w, grad_edge_vec) the outputs of
 * cgtp_conv_backward for (x, w, grad_out, edge_vec) and cotangents gg_x
 * [n_nodes][(lmax_in+1)^2][mult], gg_w [n_edges][n_paths][mult] and
 * gg_edge_vec [n_edges][3] (each nullable = zero), the call returns the
 * gradients of
 *   L = <gg_x, grad_x> + <gg_w, grad_w> + <gg_edge_vec, grad_edge_vec>
 * with respect to x (d_x), w (d_w), grad_out (d_grad_out) and the edge
 * vectors (d_edge_vec), each nullable (not computed) and overwritten.
 * Every term is one of the first-order convolutions with one argument
 * replaced (Y by (dY/dr) gg_edge_vec, x by gg_x, W by gg_w), plus
 * sum_b G_b (d2Y_b/dr2) gg_edge_vec with G the backward's harmonic gradient;
 * all run in this library's kernels.  Needs both graph views (CSR for the
 * d_grad_out sums, CSC for d_x).  When gg_edge_vec or d_edge_vec is given,
 * workspace (device, 256-byte aligned) of the size reported by
 * cgtp_conv_double_backward_workspace_size is required
 * (CGTP_ERR_WORKSPACE otherwise).
 * ------------------------------------------------------------------------- */
cgtp_status cgtp_conv_double_backward(cgtp_plan plan, int n_nodes, int n_edges,
                                      const int* row_ptr, const int* col,
                                      const int* csc_ptr, const int* csc_edge, const int* csc_dst,
                                      const float* edge_vec, const float* x, const float* w,
                                      const float* grad_out, const float* gg_x, const float* gg_w,
                                      const float* gg_edge_vec, float* d_x, float* d_w,
                                      float* d_grad_out, float* d_edge_vec, void* workspace,
                                      size_t workspace_bytes, void* stream);

/* Bytes of device workspace cgtp_uvw_forward needs for n_nodes nodes and
 * mult_out output channels (per-path messages, packed mixing matrices and
 * the GEMM's own scratch).  Mode CONV_UVW. */
cgtp_status cgtp_uvw_forward_workspace_size(cgtp_plan plan, int n_nodes, int mult_out, size_t* bytes);

/* ---------------------------------------------------------------------------
 * Fully connected ("uvw") convolution forward, the fully connected CG tensor
 * product of Equiformer ("Tensor Decomposition Networks ...", reply to
 * reviewer cmnz), mode CONV_UVW: the channelwise convolution's per-path
 * messages, summed
 * over each row but kept per path, then mixed across channels by a dense
 * matrix per path and summed into l3 blocks:
 *   t[i][p][m3][u]   = sum_{e in row i} W_e[p][u] sum C^p x[j][l1,m1][u] Y_e[l2,m2]
 *   out[i][l3,m3][v] = sum_{p: l3(p) = l3} sum_u t[i][p][m3][u] mix[p][u][v]
 * mix: device [n_paths][mult][mult_out] (paths in the plan's order);
 * out: device [n_nodes][(lmax_out+1)^2][mult_out] (overwritten).  The
 * mixing runs on the tensor cores (one GEMM per l3 block, the block's paths
 * concatenated along K) in an fp32-accurate split-bf16 mode.  mult and
 * mult_out must be multiples of 4 (CGTP_ERR_UNSUPPORTED otherwise, and when
 * the library was built without the CUTLASS headers).  workspace: device,
 * 256-byte aligned, of the size cgtp_uvw_forward_workspace_size reports
 * (CGTP_ERR_WORKSPACE otherwise).  The GEMMs of different l3 blocks run on
 * side streams of the library, forked from `stream` and joined back before
 * the call returns; the first call on a device creates them (make it before
 * any stream capture).
 * ------------------------------------------------------------------------- */
cgtp_status cgtp_uvw_forward(cgtp_plan plan, int n_nodes, int n_edges, const int* row_ptr,
                             const int* col, const float* edge_vec, const float* x, const float* w,
                             const float* mix, int mult_out, float* out, void* workspace,
                             size_t workspace_bytes, void* stream);

/* Bytes of device workspace cgtp_uvw_backward needs (with every output).
 * Mode CONV_UVW. */
cgtp_status cgtp_uvw_backward_workspace_size(cgtp_plan plan, int n_nodes, int n_edges, int mult_out,
                                             size_t* bytes);

/* ---------------------------------------------------------------------------
 * Fully connected convolution backward (mode CONV_UVW), the adjoint of
 * cgtp_uvw_forward for
 * grad_out [n_nodes][(lmax_out+1)^2][mult_out]:
 *   gt[i][p][m3][u]    = sum_v grad_out[i][l3,m3][v] mix[p][u][v]      (tensor cores)
 *   grad_mix[p][u][v]  = sum_i sum_m3 t[i][p][m3][u] grad_out[i][l3,m3][v]  (tensor cores,
 *                        t recomputed)
 * and the channelwise backward with one output gradient per path (gt):
 * grad_x [n_nodes][(lmax_in+1)^2][mult], grad_w [n_edges][n_paths][mult],
 * grad_edge_vec [n_edges][3].  Every output is nullable (not computed) and
 * overwritten.  Needs both graph views; workspace as reported by
 * cgtp_uvw_backward_workspace_size (device, 256-byte aligned).  Side streams
 * as in cgtp_uvw_forward.
 * ------------------------------------------------------------------------- */
cgtp_status cgtp_uvw_backward(cgtp_plan plan, int n_nodes, int n_edges, const int* row_ptr,
                              const int* col, const int* csc_ptr, const int* csc_edge,
                              const int* csc_dst, const float* edge_vec, const float* x,
                              const float* w, const float* mix, int mult_out,
                              const float* grad_out, float* grad_x, float* grad_w,
                              float* grad_mix, float* grad_edge_vec, void* workspace,
                              size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Per-atom forces from edge-vector gradients, F = -dE/dpos with
 * r_e = pos_src - pos_dst:  F[n] = sum_{e: dst=n} g[e] - sum_{e: src=n} g[e].
 * (Potentials predict energies and forces: "Tensor Decomposition Networks
 * ...", reply to reviewer 7Mvd, the DFT energy and force labels; the machine
 * review of "AccelNet", summary: analytic forces.  F is the negative gradient
 * of the energy through the edge vectors.)
 * Segmented sums over the CSR row and the CSC row of each node; no atomics.
 * forces: device [n_nodes][3], overwritten.
 * ------------------------------------------------------------------------- */
cgtp_status cgtp_forces(int n_nodes, int n_edges, const int* row_ptr, const int* csc_ptr,
                        const int* csc_edge, const float* grad_edge_vec, float* forces,
                        void* stream);

/* ---------------------------------------------------------------------------
 * Row gather and scatter-add: the pack and unpack of the halo exchange of a
 * graph partitioned over several GPUs (an addition of this library; the
 * pages name multi-GPU scalability without a method: "LunaTP ...",
 * abstract).  For n rows of row_floats floats (device arrays, idx int32):
 *   cgtp_gather_rows:      dst[k][:] = src[idx[k]][:]
 *   cgtp_scatter_add_rows: dst[idx[k]][:] += src[k][:]  (idx must not repeat
 *                          within one call; no atomics)
 * Float4 accesses when row_floats % 4 == 0 and src, dst are 16-byte aligned.
 * ------------------------------------------------------------------------- */
cgtp_status cgtp_gather_rows(int n, int row_floats, const int* idx, const float* src, float* dst,
                             void* stream);
cgtp_status cgtp_scatter_add_rows(int n, int row_floats, const int* idx, const float* src, float* dst,
                                  void* stream);

/* ---------------------------------------------------------------------------
 * Radial weight network (an addition of this library: the pages give none;
 * this is the per-edge weight generator of the standard workloads, the
 * Gaussian-basis MLP of NequIP-style potentials): 8 Gaussians on [0, rc]
 * (centres k*rc/7, width rc/7) -> a = phi @ W1 [8][64] -> SiLU ->
 * w = h @ W2 [64][K], no biases, K = the plan's weights per edge
 * (n_paths*mult, or mult for CONV_UVU_SHARED).  Modes CONV_UVU,
 * CONV_UVU_SHARED, CONV_UVW.  w: [n_edges][K], overwritten.
 * ------------------------------------------------------------------------- */
cgtp_status cgtp_radial_forward(cgtp_plan plan, int n_edges, const float* edge_vec, float rc,
                                const float* W1, const float* W2, float* w, void* stream);

/* dL/d edge_vec through the radial weights, ADDED to grad_edge_vec:
 * grad_edge_vec[e] += (sum_k (grad_w W2^T)_k SiLU'(a_k) (W1 dphi/dr)_k) r_e/|r_e|. */
cgtp_status cgtp_radial_backward(cgtp_plan plan, int n_edges, const float* edge_vec, float rc,
                                 const float* W1, const float* W2, const float* grad_w,
                                 float* grad_edge_vec, void* stream);

/* ---------------------------------------------------------------------------
 * Edge-free channelwise tensor product of batched pairs, mode PAIR_UVU
 * ("Tensor Decomposition Networks ...", reply to S6y1: the exact CG product,
 * timed at batch 1000 and multiplicity 128):
 *   z[b][l3,m3][u] = sum_p w[p][u] sum C^p[m1,m2,m3] x[b][l1,m1][u] y[b][l2,m2][u]
 * x: [batch][(lmax_in+1)^2][mult], y: [batch][(lmax_sh+1)^2][mult],
 * w: [n_paths][mult], z: [batch][(lmax_out+1)^2][mult] (overwritten).
 * ------------------------------------------------------------------------- */
cgtp_status cgtp_tp_forward(cgtp_plan plan, int batch, const float* x, const float* y,
                            const float* w, float* z, void* stream);

cgtp_status cgtp_tp_backward_workspace_size(cgtp_plan plan, int batch, size_t* bytes);

/* grad_x, grad_y, grad_w nullable, overwritten; grad_w (the sum over the
 * batch) needs the workspace reported by cgtp_tp_backward_workspace_size. */
cgtp_status cgtp_tp_backward(cgtp_plan plan, int batch, const float* x, const float* y,
                             const float* w, const float* grad_z, float* grad_x, float* grad_y,
                             float* grad_w, void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Allocation-free cgtp_tp_backward (an addition of this library; the paper
 * has no counterpart), mode PAIR_UVU.  For callers that cannot allocate device memory when
 * they call in: a host framework that owns all device memory through its own
 * allocator and forbids direct cudaMalloc, or a time-stepping loop that must
 * not allocate after set-up.  Same arguments and results as
 * cgtp_tp_backward, without the workspace: the grad_w partial sums live in a
 * fixed 2 MiB array inside the library (held on every device that loads it
 * until the process exits).  Allocates nothing.
 *  - Limit: tp_chunks(batch) * n_paths * mult <= 524288 floats, where the
 *    number of batch chunks is min(ceil(batch / 8), 64); so n_paths * mult
 *    <= 8192 always fits.  Larger requests return CGTP_ERR_WORKSPACE and
 *    launch nothing.
 *  - The first call on a device (with grad_w requested) looks up the array's
 *    device address (cudaGetSymbolAddress) with that device current; make
 *    that first call before any stream capture.
 *  - Every call shares the array; it keeps the last call's partial sums,
 *    which each call overwrites completely before reading.  Calls that
 *    overlap on the GPU (different streams, no ordering) race on it.
 * ------------------------------------------------------------------------- */
cgtp_status cgtp_tp_backward_noalloc(cgtp_plan plan, int batch, const float* x, const float* y,
                                     const float* w, const float* grad_z, float* grad_x, float* grad_y,
                                     float* grad_w, void* stream);

/* ---------------------------------------------------------------------------
 * CP-decomposed tensor product ("Tensor Decomposition Networks for
 * Accelerating Machine Learning Force Field Computations", reply to reviewer
 * S6y1 on the backward's complexity), mode PAIR_UVU: the low-rank surrogate
 *   z = A (B^T x (*) C^T y)                  ((*) = elementwise product)
 * of the plan's CG product, applied channelwise with factors shared by every
 * pair and channel:
 *   z[b][k][u] = sum_r A[k][r] (sum_i B[i][r] x[b][i][u]) (sum_j C[j][r] y[b][j][u]).
 * d1 = (lmax_in+1)^2, d2 = (lmax_sh+1)^2, d3 = (lmax_out+1)^2 from the plan;
 * mult from the plan.  A: [d3][rank], B: [d1][rank], C: [d2][rank] (row-major,
 * device, caller-owned); x: [batch][d1][mult], y: [batch][d2][mult],
 * z: [batch][d3][mult] (overwritten).  The factors are inputs: they are fitted
 * offline (the reply on Figure 3 fits them once, before training, by least
 * squares on batches of standard-normal inputs).
 * Errors: CGTP_ERR_INVALID_ARG for a null plan, rank < 1, batch < 0 or a null
 * pointer that the call needs; CGTP_ERR_UNSUPPORTED when the factors (and, in
 * the backward with factor gradients, the per-block staging) exceed the
 * device's shared memory per block (rank <= 256 fits every compiled shape in
 * the forward).  Nothing is launched on error.
 * ------------------------------------------------------------------------- */
cgtp_status cgtp_cp_forward(cgtp_plan plan, int rank, int batch, const float* A, const float* B,
                            const float* C, const float* x, const float* y, float* z, void* stream);

/* Workspace of cgtp_cp_backward when a factor gradient is requested:
 * ceil(batch * mult / 64) * (d1 + d2 + d3) * rank floats, rounded up to 256 bytes. */
cgtp_status cgtp_cp_backward_workspace_size(cgtp_plan plan, int rank, int batch, size_t* bytes);

/* Gradients for grad_z [batch][d3][mult]:
 *   grad_x = (g_z^T A (*) C^T y) B^T,  grad_y = (g_z^T A (*) B^T x) C^T   (per pair and channel),
 *   grad_A = sum g_z (s (*) t)^T, grad_B = sum x (q (*) t)^T, grad_C = sum y (q (*) s)^T
 * (sums over pairs and channels; s = B^T x, t = C^T y, q = A^T g_z).  Every
 * output is nullable and overwritten; the factor gradients need the workspace
 * of cgtp_cp_backward_workspace_size (CGTP_ERR_WORKSPACE otherwise) and are
 * reduced in a fixed order (bit-reproducible).  An empty batch gives zero
 * factor gradients. */
cgtp_status cgtp_cp_backward(cgtp_plan plan, int rank, int batch, const float* A, const float* B,
                             const float* C, const float* x, const float* y, const float* grad_z,
                             float* grad_x, float* grad_y, float* grad_A, float* grad_B, float* grad_C,
                             void* workspace, size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* CGTP_H */
