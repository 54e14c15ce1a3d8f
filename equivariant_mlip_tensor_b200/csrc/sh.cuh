// Real spherical harmonics (component normalisation) of an edge direction,
// and their derivative with respect to the edge vector, for l <= 4.
//
// Evaluated with the associated-Legendre three-term recurrence on the unit
// vector u = (x, y, z) and the azimuthal recurrence for
// C_m + i S_m = (x + i y)^m:
//   P_m^m = (2m-1)!!,  P_{m+1}^m = (2m+1) z P_m^m,
//   (l-m) P_l^m = (2l-1) z P_{l-1}^m - (l+m-1) P_{l-2}^m,
//   Y_l0 = K_l0 P_l^0,  Y_lm = K_lm P_l^m C_m,  Y_l,-m = K_lm P_l^m S_m,
// with K_l0 = sqrt(2l+1), K_lm = sqrt(2(2l+1)(l-m)!/(l+m)!) from constant
// memory (c_shk, filled by the host generator).  The l = 1 block is
// sqrt(3) (y, z, x).  A zero vector gives Y_00 = 1 and 0 elsewhere.
//
// This header must be included after CGTP_DEFINE_CONSTANT_TABLES.
#pragma once

namespace cgtp {

// Value plus gradient with respect to the three edge-vector components.
struct Dual3 {
  float v, d0, d1, d2;
  __device__ __forceinline__ Dual3() : v(0.f), d0(0.f), d1(0.f), d2(0.f) {}
  __device__ __forceinline__ explicit Dual3(float c) : v(c), d0(0.f), d1(0.f), d2(0.f) {}
  __device__ __forceinline__ Dual3(float a, float b, float c, float d) : v(a), d0(b), d1(c), d2(d) {}
};
__device__ __forceinline__ Dual3 operator+(const Dual3& a, const Dual3& b) {
  return Dual3(a.v + b.v, a.d0 + b.d0, a.d1 + b.d1, a.d2 + b.d2);
}
__device__ __forceinline__ Dual3 operator-(const Dual3& a, const Dual3& b) {
  return Dual3(a.v - b.v, a.d0 - b.d0, a.d1 - b.d1, a.d2 - b.d2);
}
__device__ __forceinline__ Dual3 operator*(const Dual3& a, const Dual3& b) {
  return Dual3(a.v * b.v, fmaf(a.v, b.d0, a.d0 * b.v), fmaf(a.v, b.d1, a.d1 * b.v),
               fmaf(a.v, b.d2, a.d2 * b.v));
}
__device__ __forceinline__ Dual3 operator*(float s, const Dual3& a) {
  return Dual3(s * a.v, s * a.d0, s * a.d1, s * a.d2);
}

// Value plus derivative along one direction q: f + t q.grad f (first order).
struct Dual1 {
  float v, e;
  __device__ __forceinline__ Dual1() : v(0.f), e(0.f) {}
  __device__ __forceinline__ explicit Dual1(float c) : v(c), e(0.f) {}
  __device__ __forceinline__ Dual1(float a, float b) : v(a), e(b) {}
};
__device__ __forceinline__ Dual1 operator+(const Dual1& a, const Dual1& b) { return Dual1(a.v + b.v, a.e + b.e); }
__device__ __forceinline__ Dual1 operator-(const Dual1& a, const Dual1& b) { return Dual1(a.v - b.v, a.e - b.e); }
__device__ __forceinline__ Dual1 operator*(const Dual1& a, const Dual1& b) {
  return Dual1(a.v * b.v, fmaf(a.v, b.e, a.e * b.v));
}
__device__ __forceinline__ Dual1 operator*(float s, const Dual1& a) { return Dual1(s * a.v, s * a.e); }

// Gradient with respect to the edge vector of a Dual1-valued function: the
// t-part of component k is (d2f/dr2 q)_k, a Hessian-vector product.
struct HDual {
  Dual1 v, d0, d1, d2;
  __device__ __forceinline__ HDual() {}
  __device__ __forceinline__ explicit HDual(float c) : v(c) {}
  __device__ __forceinline__ HDual(Dual1 a, Dual1 b, Dual1 c, Dual1 d) : v(a), d0(b), d1(c), d2(d) {}
};
__device__ __forceinline__ HDual operator+(const HDual& a, const HDual& b) {
  return HDual(a.v + b.v, a.d0 + b.d0, a.d1 + b.d1, a.d2 + b.d2);
}
__device__ __forceinline__ HDual operator-(const HDual& a, const HDual& b) {
  return HDual(a.v - b.v, a.d0 - b.d0, a.d1 - b.d1, a.d2 - b.d2);
}
__device__ __forceinline__ HDual operator*(const HDual& a, const HDual& b) {
  return HDual(a.v * b.v, a.v * b.d0 + a.d0 * b.v, a.v * b.d1 + a.d1 * b.v, a.v * b.d2 + a.d2 * b.v);
}
__device__ __forceinline__ HDual operator*(float s, const HDual& a) {
  return HDual(s * a.v, s * a.d0, s * a.d1, s * a.d2);
}

__device__ __forceinline__ float scal(float c) { return c; }

template <class S>
__device__ __forceinline__ S mk(float c) { return S(c); }

constexpr float dfact(int m) {  // (2m-1)!!
  float r = 1.f;
  for (int k = 2 * m - 1; k > 1; k -= 2) r *= float(k);
  return r;
}

// Y[(LS+1)^2] of the unit vector (x, y, z); S is float or Dual3.
template <int LS, class S>
static __device__ __forceinline__ void sh_unit(const S& x, const S& y, const S& z, S (&Y)[(LS + 1) * (LS + 1)]) {
  S Cm[LS + 1], Sm[LS + 1];
  Cm[0] = mk<S>(1.f);
  Sm[0] = mk<S>(0.f);
#pragma unroll
  for (int m = 1; m <= LS; ++m) {
    Cm[m] = x * Cm[m - 1] - y * Sm[m - 1];
    Sm[m] = x * Sm[m - 1] + y * Cm[m - 1];
  }
  S P[LS + 1][LS + 1];
#pragma unroll
  for (int m = 0; m <= LS; ++m) {
    P[m][m] = mk<S>(dfact(m));
    if (m + 1 <= LS) P[m + 1][m] = float(2 * m + 1) * (z * P[m][m]);
#pragma unroll
    for (int l = m + 2; l <= LS; ++l)
      P[l][m] = (1.f / float(l - m)) * (float(2 * l - 1) * (z * P[l - 1][m]) - float(l + m - 1) * P[l - 2][m]);
  }
#pragma unroll
  for (int l = 0; l <= LS; ++l) {
    Y[l * l + l] = c_shk[shk_index(l, 0)] * P[l][0];
#pragma unroll
    for (int m = 1; m <= l; ++m) {
      const S kp = c_shk[shk_index(l, m)] * P[l][m];
      Y[l * l + l + m] = kp * Cm[m];
      Y[l * l + l - m] = kp * Sm[m];
    }
  }
}

// Harmonics of edge vector (vx, vy, vz) in fp32.
template <int LS>
static __device__ __forceinline__ void sh_of_vec(float vx, float vy, float vz, float (&Y)[(LS + 1) * (LS + 1)]) {
  const float r2 = fmaf(vx, vx, fmaf(vy, vy, vz * vz));
  if (r2 > 0.f) {
    const float inv = rsqrtf(r2);
    sh_unit<LS, float>(vx * inv, vy * inv, vz * inv, Y);
  } else {
#pragma unroll
    for (int k = 0; k < (LS + 1) * (LS + 1); ++k) Y[k] = 0.f;
    Y[0] = 1.f;
  }
}

// Harmonics and their gradients with respect to the raw edge vector.
template <int LS>
static __device__ __forceinline__ void sh_grad_of_vec(float vx, float vy, float vz,
                                               Dual3 (&Y)[(LS + 1) * (LS + 1)]) {
  const float r2 = fmaf(vx, vx, fmaf(vy, vy, vz * vz));
  if (r2 > 0.f) {
    const Dual3 X(vx, 1.f, 0.f, 0.f), Yv(vy, 0.f, 1.f, 0.f), Z(vz, 0.f, 0.f, 1.f);
    const float r = sqrtf(r2);
    const float inv = 1.f / r;
    // d(1/r)/dv = -v / r^3
    const float g = -inv * inv * inv;
    const Dual3 invd(inv, g * vx, g * vy, g * vz);
    sh_unit<LS, Dual3>(X * invd, Yv * invd, Z * invd, Y);
  } else {
#pragma unroll
    for (int k = 0; k < (LS + 1) * (LS + 1); ++k) Y[k] = Dual3(0.f);
    Y[0] = Dual3(1.f);
  }
}

// Directional derivative (dY/dr) q of the harmonics: Y[b].e for every b.
template <int LS>
static __device__ __forceinline__ void sh_dir_of_vec(float vx, float vy, float vz, float qx, float qy, float qz,
                                                     Dual1 (&Y)[(LS + 1) * (LS + 1)]) {
  const float r2 = fmaf(vx, vx, fmaf(vy, vy, vz * vz));
  if (r2 > 0.f) {
    const float inv = rsqrtf(r2);
    // d(r2^-1/2) = -r2^-3/2 (v . q) along q
    const float vq = fmaf(vx, qx, fmaf(vy, qy, vz * qz));
    const Dual1 invd(inv, -inv * inv * inv * vq);
    sh_unit<LS, Dual1>(Dual1(vx, qx) * invd, Dual1(vy, qy) * invd, Dual1(vz, qz) * invd, Y);
  } else {
#pragma unroll
    for (int k = 0; k < (LS + 1) * (LS + 1); ++k) Y[k] = Dual1(0.f);
    Y[0] = Dual1(1.f);
  }
}

// Harmonics with their gradient and the Hessian-vector product along q:
// Y[b].dk.v = dY_b/dr_k and Y[b].dk.e = (d2Y_b/dr2 q)_k.
template <int LS>
static __device__ __forceinline__ void sh_hess_of_vec(float vx, float vy, float vz, float qx, float qy, float qz,
                                                      HDual (&Y)[(LS + 1) * (LS + 1)]) {
  const float r2 = fmaf(vx, vx, fmaf(vy, vy, vz * vz));
  if (r2 > 0.f) {
    const Dual1 one(1.f), zero(0.f);
    const HDual X(Dual1(vx, qx), one, zero, zero), Yv(Dual1(vy, qy), zero, one, zero),
        Z(Dual1(vz, qz), zero, zero, one);
    // s = r2 as an HDual, then s^-1/2 by the chain rule at both orders:
    // f = s^-1/2, f' = -s^-3/2 / 2, f'' = 3 s^-5/2 / 4, each carried along q.
    const HDual s = X * X + Yv * Yv + Z * Z;
    const float inv = rsqrtf(s.v.v);
    const float f0 = inv, f1 = -0.5f * inv * inv * inv, f2 = 0.75f * inv * inv * inv * inv * inv;
    const Dual1 fs(f0, f1 * s.v.e), dfs(f1, f2 * s.v.e);
    const HDual invd(fs, dfs * s.d0, dfs * s.d1, dfs * s.d2);
    sh_unit<LS, HDual>(X * invd, Yv * invd, Z * invd, Y);
  } else {
#pragma unroll
    for (int k = 0; k < (LS + 1) * (LS + 1); ++k) Y[k] = HDual(0.f);
    Y[0] = HDual(1.f);
  }
}

// Harmonics of edge e: the caller's per-edge values when given, else Y(edge_vec[e]).
template <int LS>
static __device__ __forceinline__ void edge_sh(const float* __restrict__ sh, const float* __restrict__ edge_vec,
                                               long long e, float (&Y)[(LS + 1) * (LS + 1)]) {
  constexpr int NS = (LS + 1) * (LS + 1);
  if (sh != nullptr) {
#pragma unroll
    for (int b = 0; b < NS; ++b) Y[b] = __ldg(sh + e * NS + b);
  } else {
    sh_of_vec<LS>(__ldg(edge_vec + 3 * e), __ldg(edge_vec + 3 * e + 1), __ldg(edge_vec + 3 * e + 2), Y);
  }
}

}  // namespace cgtp
