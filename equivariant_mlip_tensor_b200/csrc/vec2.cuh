// Channel-vector FMAs for sm_100a: two channels per packed f32x2 FMA
// (__ffma2_rn, each lane rounded like fmaf) when the vector width is even.
#pragma once
#include <cuda_runtime.h>

namespace cgtp {

// acc[c] += s v[c]
template <int VEC>
__device__ __forceinline__ void axpy(float (&acc)[VEC], float s, const float (&v)[VEC]) {
  if constexpr (VEC % 2 == 0) {
    const float2 s2 = make_float2(s, s);
#pragma unroll
    for (int c = 0; c < VEC; c += 2) {
      const float2 r = __ffma2_rn(s2, make_float2(v[c], v[c + 1]), make_float2(acc[c], acc[c + 1]));
      acc[c] = r.x;
      acc[c + 1] = r.y;
    }
  } else {
#pragma unroll
    for (int c = 0; c < VEC; ++c) acc[c] = fmaf(s, v[c], acc[c]);
  }
}

// acc[c] += a[c] b[c]
template <int VEC>
__device__ __forceinline__ void vfma(float (&acc)[VEC], const float (&a)[VEC], const float (&b)[VEC]) {
  if constexpr (VEC % 2 == 0) {
#pragma unroll
    for (int c = 0; c < VEC; c += 2) {
      const float2 r =
          __ffma2_rn(make_float2(a[c], a[c + 1]), make_float2(b[c], b[c + 1]), make_float2(acc[c], acc[c + 1]));
      acc[c] = r.x;
      acc[c + 1] = r.y;
    }
  } else {
#pragma unroll
    for (int c = 0; c < VEC; ++c) acc[c] = fmaf(a[c], b[c], acc[c]);
  }
}

// out[c] = a[c] b[c]
template <int VEC>
__device__ __forceinline__ void vmul(float (&out)[VEC], const float (&a)[VEC], const float (&b)[VEC]) {
  if constexpr (VEC % 2 == 0) {
#pragma unroll
    for (int c = 0; c < VEC; c += 2) {
      const float2 r = __fmul2_rn(make_float2(a[c], a[c + 1]), make_float2(b[c], b[c + 1]));
      out[c] = r.x;
      out[c + 1] = r.y;
    }
  } else {
#pragma unroll
    for (int c = 0; c < VEC; ++c) out[c] = a[c] * b[c];
  }
}

// sum_c a[c] b[c] (even and odd channels summed separately, then added, for even VEC)
template <int VEC>
__device__ __forceinline__ float vdot(const float (&a)[VEC], const float (&b)[VEC]) {
  if constexpr (VEC % 2 == 0) {
    float2 s = __fmul2_rn(make_float2(a[0], a[1]), make_float2(b[0], b[1]));
#pragma unroll
    for (int c = 2; c < VEC; c += 2) s = __ffma2_rn(make_float2(a[c], a[c + 1]), make_float2(b[c], b[c + 1]), s);
    return s.x + s.y;
  } else {
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < VEC; ++c) s = fmaf(a[c], b[c], s);
    return s;
  }
}

}  // namespace cgtp
