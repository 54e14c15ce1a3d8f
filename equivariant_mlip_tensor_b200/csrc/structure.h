// Compile-time structure of the real-basis Clebsch-Gordan paths.
//
// Shared by the host table generator and the kernels so that both agree on
// where every coefficient lives.  The real-basis selection rules used here
// follow from the complex ones (|l1-l2| <= l3 <= l1+l2, m3 = m1+m2; "Tensor
// Decomposition Networks ...", reply to reviewer S6y1) and the change of
// basis: a real coefficient can be nonzero only if
//   |m3| is |m1|+|m2| or ||m1|-|m2||, and
//   the number of negative m's has the parity of l1+l2+l3
// (the real basis is even/odd under y -> -y for m >= 0 / m < 0).  The host
// generator checks that every coefficient outside this pattern vanishes.
#pragma once

#if defined(__CUDACC__)
#define CGTP_HD __host__ __device__
#else
#define CGTP_HD
#endif

namespace cgtp {

constexpr int kLmaxTab = 4;   // every path with l1, l2, l3 <= 4 is tabulated
constexpr int kMaxPaths = 72;

CGTP_HD constexpr int iabs(int a) { return a < 0 ? -a : a; }

CGTP_HD constexpr bool triangle(int l1, int l2, int l3) {
  return iabs(l1 - l2) <= l3 && l3 <= l1 + l2;
}

// Structural nonzero pattern of the real CG block of path (l1, l2, l3);
// m's are signed (-l..l).
CGTP_HD constexpr bool cg_allowed(int l1, int l2, int l3, int m1, int m2, int m3) {
  if (!triangle(l1, l2, l3)) return false;
  if (iabs(m1) > l1 || iabs(m2) > l2 || iabs(m3) > l3) return false;
  const int a = iabs(m1), b = iabs(m2), c = iabs(m3);
  if (!(c == a + b || c == iabs(a - b))) return false;
  const int neg = (m1 < 0 ? 1 : 0) + (m2 < 0 ? 1 : 0) + (m3 < 0 ? 1 : 0);
  return (neg & 1) == ((l1 + l2 + l3) & 1);
}

CGTP_HD constexpr int path_entries(int l1, int l2, int l3) {
  int n = 0;
  for (int m1 = -l1; m1 <= l1; ++m1)
    for (int m2 = -l2; m2 <= l2; ++m2)
      for (int m3 = -l3; m3 <= l3; ++m3) n += cg_allowed(l1, l2, l3, m1, m2, m3) ? 1 : 0;
  return n;
}

// Offsets of every tabulated path in the global coefficient table
// (paths in lexicographic (l1, l2, l3) order, entries in lexicographic
// (m1, m2, m3) order).
struct TableLayout {
  int base[kLmaxTab + 1][kLmaxTab + 1][kLmaxTab + 1];
  int total;
};

CGTP_HD constexpr TableLayout make_table_layout() {
  TableLayout t{};
  int off = 0;
  for (int a = 0; a <= kLmaxTab; ++a)
    for (int b = 0; b <= kLmaxTab; ++b)
      for (int c = 0; c <= kLmaxTab; ++c) {
        t.base[a][b][c] = off;
        if (triangle(a, b, c)) off += path_entries(a, b, c);
      }
  t.total = off;
  return t;
}

constexpr TableLayout kTable = make_table_layout();
constexpr int kTableSize = kTable.total;

// Position of coefficient (m1, m2, m3) of path (l1, l2, l3) in the table, or -1.
CGTP_HD constexpr int table_index(int l1, int l2, int l3, int m1, int m2, int m3) {
  if (!cg_allowed(l1, l2, l3, m1, m2, m3)) return -1;
  int k = 0;
  for (int a = -l1; a <= l1; ++a)
    for (int b = -l2; b <= l2; ++b)
      for (int c = -l3; c <= l3; ++c) {
        if (!cg_allowed(l1, l2, l3, a, b, c)) continue;
        if (a == m1 && b == m2 && c == m3) return kTable.base[l1][l2][l3] + k;
        ++k;
      }
  return -1;
}

// Spherical-harmonic normalisation constants K_lm (m >= 0), index l(l+1)/2 + m.
constexpr int kShkSize = (kLmaxTab + 1) * (kLmaxTab + 2) / 2;
CGTP_HD constexpr int shk_index(int l, int m) { return l * (l + 1) / 2 + m; }

// The path list of one irreps shape, and the per-edge matrices
// T^p[m1][m3] = sum_m2 C^p[m1,m2,m3] Y[l2,m2] packed per path in (m3, m1)
// order, each path's block padded to a multiple of 4 floats.
struct PathData {
  int np;
  int l1[kMaxPaths], l2[kMaxPaths], l3[kMaxPaths];
  int tbase[kMaxPaths + 1];   // padded start of each path's T block
  int tcount[kMaxPaths];      // structural T entries of the path
  int nnz;                    // structural CG entries over all paths
  int by_l2[kMaxPaths];       // path numbers sorted by (l2, l1, l3)
  bool last_of_l2[kMaxPaths]; // by_l2[k] is the last path with its l2
};

CGTP_HD constexpr bool t_allowed(int l1, int l2, int l3, int m1, int m3) {
  for (int m2 = -l2; m2 <= l2; ++m2)
    if (cg_allowed(l1, l2, l3, m1, m2, m3)) return true;
  return false;
}

CGTP_HD constexpr PathData make_paths(int LI, int LS, int LO) {
  PathData d{};
  int p = 0, off = 0, nnz = 0;
  for (int a = 0; a <= LI; ++a)
    for (int b = 0; b <= LS; ++b)
      for (int c = iabs(a - b); c <= (a + b < LO ? a + b : LO); ++c) {
        d.l1[p] = a;
        d.l2[p] = b;
        d.l3[p] = c;
        d.tbase[p] = off;
        int cnt = 0;
        for (int m3 = -c; m3 <= c; ++m3)
          for (int m1 = -a; m1 <= a; ++m1) cnt += t_allowed(a, b, c, m1, m3) ? 1 : 0;
        d.tcount[p] = cnt;
        off += (cnt + 3) / 4 * 4;
        nnz += path_entries(a, b, c);
        ++p;
      }
  d.np = p;
  d.tbase[p] = off;
  d.nnz = nnz;
  int k = 0;
  for (int b = 0; b <= LS; ++b)
    for (int q = 0; q < p; ++q)
      if (d.l2[q] == b) d.by_l2[k++] = q;
  for (int q = 0; q < p; ++q) d.last_of_l2[q] = (q + 1 == p) || d.l2[d.by_l2[q + 1]] != d.l2[d.by_l2[q]];
  return d;
}

template <int LI_, int LS_, int LO_>
struct PathSet {
  static constexpr int LI = LI_, LS = LS_, LO = LO_;
  static constexpr int NI = (LI + 1) * (LI + 1);
  static constexpr int NS = (LS + 1) * (LS + 1);
  static constexpr int NO = (LO + 1) * (LO + 1);
  static constexpr PathData D = make_paths(LI, LS, LO);
  static constexpr int NP = D.np;
  static constexpr int NT = D.tbase[D.np];  // floats of one edge's T (padded)

  // Index of T^p[m1][m3] (signed m) in one edge's T, or -1 if structurally zero.
  CGTP_HD static constexpr int t_index(int p, int m1, int m3) {
    const int a = D.l1[p], b = D.l2[p], c = D.l3[p];
    if (!t_allowed(a, b, c, m1, m3)) return -1;
    int k = 0;
    for (int q3 = -c; q3 <= c; ++q3)
      for (int q1 = -a; q1 <= a; ++q1) {
        if (!t_allowed(a, b, c, q1, q3)) continue;
        if (q1 == m1 && q3 == m3) return D.tbase[p] + k;
        ++k;
      }
    return -1;
  }

  // (m1, m3) of the k-th structural T entry of path p (k < tcount[p]).
  CGTP_HD static constexpr int t_entry_m1(int p, int k) {
    const int a = D.l1[p], b = D.l2[p], c = D.l3[p];
    int n = 0;
    for (int q3 = -c; q3 <= c; ++q3)
      for (int q1 = -a; q1 <= a; ++q1) {
        if (!t_allowed(a, b, c, q1, q3)) continue;
        if (n == k) return q1;
        ++n;
      }
    return 0;
  }
  CGTP_HD static constexpr int t_entry_m3(int p, int k) {
    const int a = D.l1[p], b = D.l2[p], c = D.l3[p];
    int n = 0;
    for (int q3 = -c; q3 <= c; ++q3)
      for (int q1 = -a; q1 <= a; ++q1) {
        if (!t_allowed(a, b, c, q1, q3)) continue;
        if (n == k) return q3;
        ++n;
      }
    return 0;
  }
};

}  // namespace cgtp
