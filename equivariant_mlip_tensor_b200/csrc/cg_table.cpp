// Host generator of the real-basis Clebsch-Gordan coefficients (fp64).
//
// Selection rules: "Tensor Decomposition Networks ...", reply to reviewer
// S6y1 (|l1-l2| <= l3 <= l1+l2, m3 = m1+m2).  The coefficients are built
// without any closed-form sum: the coupled states |J M> of j1 x j2 are
// constructed in the product basis |m1 m2> by the angular-momentum lowering
// operator J- = J1- + J2-, starting from the stretched state
// |j1+j2, j1+j2> = |j1 j1>|j2 j2>.  Each lower J starts from the unique
// (up to sign) vector of the M = J subspace orthogonal to all higher J, with
// the Condon-Shortley sign <j1 j1, j2 J-j1 | J J> > 0.  The complex-basis
// coefficients are then carried into the real basis
//   real m > 0: (Y^{-m} + (-1)^m Y^m)/sqrt2, m = 0: Y^0,
//   real m < 0: i (Y^m - (-1)^m Y^{-m})/sqrt2,
// as C_r[a,b,c] = sum Q3[c,M] C[m1,m2,M] conj(Q1[a,m1]) conj(Q2[b,m2]);
// each path is then purely real or purely imaginary, and the real part is
// kept when it is nonzero, else the imaginary part.
#include "cg_table.h"

#include <cmath>
#include <complex>
#include <vector>

#include "structure.h"

namespace cgtp {
namespace {

using cd = std::complex<double>;

// Coupled states of j1 x j2: states[J][M + J] is a vector over (m1, m2),
// index (m1 + j1) * (2 j2 + 1) + (m2 + j2).
struct Coupling {
  int j1, j2;
  std::vector<std::vector<std::vector<double>>> states;  // [J][M+J][dim]
};

int product_index(int j1, int j2, int m1, int m2) { return (m1 + j1) * (2 * j2 + 1) + (m2 + j2); }

Coupling couple(int j1, int j2) {
  Coupling cp{j1, j2, {}};
  const int dim = (2 * j1 + 1) * (2 * j2 + 1);
  const int Jmax = j1 + j2, Jmin = j1 > j2 ? j1 - j2 : j2 - j1;
  cp.states.assign(Jmax + 1, {});
  for (int J = Jmax; J >= Jmin; --J) {
    std::vector<std::vector<double>>& st = cp.states[J];
    st.assign(2 * J + 1, std::vector<double>(dim, 0.0));
    // top state |J, J>
    std::vector<double> v(dim, 0.0);
    v[product_index(j1, j2, j1, J - j1)] = 1.0;
    for (int Jp = J + 1; Jp <= Jmax; ++Jp) {  // Gram-Schmidt against higher J at M = J
      const std::vector<double>& u = cp.states[Jp][J + Jp];
      double dot = 0.0;
      for (int k = 0; k < dim; ++k) dot += u[k] * v[k];
      for (int k = 0; k < dim; ++k) v[k] -= dot * u[k];
    }
    double nrm = 0.0;
    for (int k = 0; k < dim; ++k) nrm += v[k] * v[k];
    nrm = std::sqrt(nrm);
    const double sgn = v[product_index(j1, j2, j1, J - j1)] >= 0.0 ? 1.0 : -1.0;
    for (int k = 0; k < dim; ++k) v[k] *= sgn / nrm;
    st[2 * J] = v;
    // lower: |J, M-1> = J- |J, M> / sqrt(J(J+1) - M(M-1))
    for (int M = J; M > -J; --M) {
      const std::vector<double>& cur = st[M + J];
      std::vector<double> nxt(dim, 0.0);
      for (int m1 = -j1; m1 <= j1; ++m1)
        for (int m2 = -j2; m2 <= j2; ++m2) {
          const double c = cur[product_index(j1, j2, m1, m2)];
          if (c == 0.0) continue;
          if (m1 > -j1)
            nxt[product_index(j1, j2, m1 - 1, m2)] += c * std::sqrt(double(j1 * (j1 + 1) - m1 * (m1 - 1)));
          if (m2 > -j2)
            nxt[product_index(j1, j2, m1, m2 - 1)] += c * std::sqrt(double(j2 * (j2 + 1) - m2 * (m2 - 1)));
        }
      const double s = 1.0 / std::sqrt(double(J * (J + 1) - M * (M - 1)));
      for (int k = 0; k < dim; ++k) nxt[k] *= s;
      st[M - 1 + J] = nxt;
    }
  }
  return cp;
}

// Q_l[real m + l][complex m + l]
std::vector<cd> real_basis(int l) {
  const int d = 2 * l + 1;
  std::vector<cd> Q(d * d, cd(0.0, 0.0));
  const double r = 1.0 / std::sqrt(2.0);
  for (int m = -l; m <= l; ++m) {
    const int row = m + l;
    const double par = (m % 2 == 0) ? 1.0 : -1.0;  // (-1)^m
    if (m > 0) {
      Q[row * d + (-m + l)] = cd(r, 0.0);
      Q[row * d + (m + l)] = cd(par * r, 0.0);
    } else if (m == 0) {
      Q[row * d + l] = cd(1.0, 0.0);
    } else {
      Q[row * d + (m + l)] = cd(0.0, r);
      Q[row * d + (-m + l)] = cd(0.0, -par * r);
    }
  }
  return Q;
}

}  // namespace

bool real_cg_block(int l1, int l2, int l3, double* out, double* discarded) {
  const int d1 = 2 * l1 + 1, d2 = 2 * l2 + 1, d3 = 2 * l3 + 1;
  for (int k = 0; k < d1 * d2 * d3; ++k) out[k] = 0.0;
  if (discarded) *discarded = 0.0;
  if (l1 < 0 || l2 < 0 || l3 < 0 || !triangle(l1, l2, l3)) return true;
  const Coupling cp = couple(l1, l2);
  const std::vector<std::vector<double>>& st = cp.states[l3];
  // complex C[m1][m2][M]
  std::vector<double> C(d1 * d2 * d3, 0.0);
  for (int M = -l3; M <= l3; ++M)
    for (int m1 = -l1; m1 <= l1; ++m1)
      for (int m2 = -l2; m2 <= l2; ++m2)
        C[((m1 + l1) * d2 + (m2 + l2)) * d3 + (M + l3)] = st[M + l3][product_index(l1, l2, m1, m2)];
  const std::vector<cd> Q1 = real_basis(l1), Q2 = real_basis(l2), Q3 = real_basis(l3);
  std::vector<cd> R(d1 * d2 * d3, cd(0.0, 0.0));
  for (int a = 0; a < d1; ++a)
    for (int b = 0; b < d2; ++b)
      for (int c = 0; c < d3; ++c) {
        cd s(0.0, 0.0);
        for (int i = 0; i < d1; ++i) {
          const cd q1 = std::conj(Q1[a * d1 + i]);
          if (q1 == cd(0.0, 0.0)) continue;
          for (int j = 0; j < d2; ++j) {
            const cd q2 = std::conj(Q2[b * d2 + j]);
            if (q2 == cd(0.0, 0.0)) continue;
            for (int M = 0; M < d3; ++M) {
              const double cv = C[(i * d2 + j) * d3 + M];
              if (cv == 0.0) continue;
              s += Q3[c * d3 + M] * cv * q1 * q2;
            }
          }
        }
        R[(a * d2 + b) * d3 + c] = s;
      }
  double max_re = 0.0, max_im = 0.0;
  for (const cd& v : R) {
    max_re = std::fmax(max_re, std::fabs(v.real()));
    max_im = std::fmax(max_im, std::fabs(v.imag()));
  }
  const bool take_re = max_re > 1e-12;
  for (int k = 0; k < d1 * d2 * d3; ++k) {
    const double v = take_re ? R[k].real() : R[k].imag();
    out[k] = std::fabs(v) < 1e-15 ? 0.0 : v;
  }
  if (discarded) *discarded = take_re ? max_im : max_re;
  return true;
}

int build_constant_tables(float* cg_table, float* shk) {
  std::vector<double> blk;
  for (int a = 0; a <= kLmaxTab; ++a)
    for (int b = 0; b <= kLmaxTab; ++b)
      for (int c = 0; c <= kLmaxTab; ++c) {
        if (!triangle(a, b, c)) continue;
        const int d1 = 2 * a + 1, d2 = 2 * b + 1, d3 = 2 * c + 1;
        blk.assign(d1 * d2 * d3, 0.0);
        double disc = 0.0;
        real_cg_block(a, b, c, blk.data(), &disc);
        if (disc > 1e-12) return 1;
        // unitary columns: sum_{a,b} C[.,.,c] C[.,.,c'] = delta
        for (int c1 = 0; c1 < d3; ++c1)
          for (int c2 = 0; c2 < d3; ++c2) {
            double s = 0.0;
            for (int i = 0; i < d1 * d2; ++i) s += blk[i * d3 + c1] * blk[i * d3 + c2];
            if (std::fabs(s - (c1 == c2 ? 1.0 : 0.0)) > 1e-12) return 2;
          }
        for (int m1 = -a; m1 <= a; ++m1)
          for (int m2 = -b; m2 <= b; ++m2)
            for (int m3 = -c; m3 <= c; ++m3) {
              const double v = blk[((m1 + a) * d2 + (m2 + b)) * d3 + (m3 + c)];
              const int idx = table_index(a, b, c, m1, m2, m3);
              if (idx < 0) {
                if (std::fabs(v) > 1e-12) return 3;  // outside the structural pattern
              } else {
                cg_table[idx] = static_cast<float>(v);
              }
            }
      }
  // K_l0 = sqrt(2l+1), K_lm = sqrt(2 (2l+1) (l-m)! / (l+m)!)
  for (int l = 0; l <= kLmaxTab; ++l)
    for (int m = 0; m <= l; ++m) {
      double ratio = 1.0;
      for (int k = l - m + 1; k <= l + m; ++k) ratio /= double(k);
      const double K = m == 0 ? std::sqrt(2.0 * l + 1.0) : std::sqrt(2.0 * (2.0 * l + 1.0) * ratio);
      shk[shk_index(l, m)] = static_cast<float>(K);
    }
  return 0;
}

}  // namespace cgtp
