// Per-element RG-LRU gate arithmetic, "Griffin：将门控线性循环与局部注意力混合以实现
// 高效的语言模型", §实门线性循环单元 (RG-LRU), Eq. (1)–(4):
//   r = σ(z_a), i = σ(z_x), log a_t = c r log σ(Λ), a_t = exp(log a_t),
//   b_t = √(1 − a_t²) · i · u,  so that h_t = a_t h_{t-1} + b_t.
// The decay is taken in log space as the page prescribes for numerical stability:
// log σ(Λ) = −softplus(−Λ) is precomputed per channel (cla = c · log σ(Λ)), and
// 1 − a_t² is formed as −expm1(2 log a_t), which keeps its relative accuracy when
// a_t is close to 1 (a^c ∈ [0.9, 0.999] puts a_t within 1.3e-4 of 1).
#pragma once
#include <cuda_runtime.h>

namespace rglru {

constexpr float kDecayC = 8.0f;       // the constant c of Eq. (3)
constexpr float kLog2e = 1.4426950408889634f;

// c · log σ(Λ) = −c · softplus(−Λ), written so that no intermediate overflows.
__device__ __forceinline__ float decay_log_coeff(float lam) {
  const float sp = fmaxf(-lam, 0.0f) + log1pf(expf(-fabsf(lam)));
  return -kDecayC * sp;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rsqrt_approx(float x) {
  float y;
  asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// −expm1(x) for x ∈ (−0.25, 0]: the Taylor series of e^x − 1 about 0 to degree 7,
// −x (1 + x/2 + x²/6 + x³/24 + x⁴/120 + x⁵/720 + x⁶/5040); the first omitted term is
// below 2e-9 of the result on this interval.
__device__ __forceinline__ float neg_expm1_small(float x) {
  float p = 1.0f / 5040.0f;
  p = fmaf(p, x, 1.0f / 720.0f);
  p = fmaf(p, x, 1.0f / 120.0f);
  p = fmaf(p, x, 1.0f / 24.0f);
  p = fmaf(p, x, 1.0f / 6.0f);
  p = fmaf(p, x, 0.5f);
  p = fmaf(p, x, 1.0f);
  return -x * p;
}

// Accurate form (float32 IO): CUDA's expf/expm1f/sqrtf and IEEE division.
__device__ __forceinline__ void gate_accurate(float za, float zx, float cla, float u, float& a_t, float& b_t) {
  const float r = 1.0f / (1.0f + expf(-za));
  const float la = r * cla;
  a_t = expf(la);
  const float q = -expm1f(2.0f * la);
  const float i = 1.0f / (1.0f + expf(-zx));
  b_t = sqrtf(q) * i * u;
}

// Fast form (bf16 IO): hardware ex2/rcp/rsqrt approximations (relative error ~1e-7),
// five MUFU operations per element. √(1 − a_t²)·i is formed as q·rsqrt(q (1 + e^{−z_x})²)
// with q = 1 − a_t², which saves the reciprocal of the input gate.
__device__ __forceinline__ void gate_fast(float za, float zx, float cla, float u, float& a_t, float& b_t) {
  const float ea = ex2_approx(-za * kLog2e);
  const float r = rcp_approx(1.0f + ea);
  const float la = r * cla;
  a_t = ex2_approx(la * kLog2e);
  const float x2 = 2.0f * la;
  const float q = (x2 > -0.25f) ? neg_expm1_small(x2) : fmaf(-a_t, a_t, 1.0f);
  const float ex = ex2_approx(-zx * kLog2e);
  const float t1 = 1.0f + ex;
  const float d = q * t1 * t1;
  const float mi = (q > 0.0f) ? q * rsqrt_approx(fmaxf(d, 1e-30f)) : 0.0f;
  b_t = mi * u;
}

template <bool kAccurate>
__device__ __forceinline__ void gate(float za, float zx, float cla, float u, float& a_t, float& b_t) {
  if constexpr (kAccurate) gate_accurate(za, zx, cla, u, a_t, b_t);
  else gate_fast(za, zx, cla, u, a_t, b_t);
}

// GeLU, exact erf form x·Φ(x) (the block's second branch).
__device__ __forceinline__ float gelu_exact(float g) { return 0.5f * g * (1.0f + erff(g * 0.70710678118654752f)); }

}  // namespace rglru
