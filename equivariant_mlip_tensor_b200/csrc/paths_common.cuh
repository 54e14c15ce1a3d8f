// Layout and chunk planning of the per-path messages of the fully connected
// convolution (conv_paths.cu).
//
// The messages of each path are kept apart in blocks by l3: block l3 holds
// [node][m3][rank][u] for the paths of that l3 in (l2, path number) order,
// and the blocks follow one another in increasing l3.  Include after
// conv_common.cuh.
#pragma once

namespace cgtp {

// place of path p among the paths of its l3 block
template <class PS>
constexpr int l3_rank(int p) {
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

// Chunks of same-key paths (the planner of conv_common.cuh) that also keep
// at most max_rows output rows (sum of 2 l3 + 1 over the chunk's paths), for
// kernels that hold one block of accumulators per path.
template <class PS>
constexpr ChunkPlan make_chunk_plan_rows(int kind, int vec, bool gy, int budget, int max_rows) {
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
    c.key[c.n] = key;
    c.first[c.n] = start;
    c.count[c.n] = end - start;
    c.first_of_key[c.n] = c.n == 0 || c.key[c.n - 1] != key;
    ++c.n;
    start = end;
  }
  return c;
}

template <class PS, int KIND, int VEC, bool GY, int BUDGET, int MAX_ROWS>
struct PlanRows {
  static constexpr ChunkPlan P = make_chunk_plan_rows<PS>(KIND, VEC, GY, BUDGET, MAX_ROWS);
  static constexpr int N = P.n;
};

}  // namespace cgtp
