// Width-4 causal depthwise Conv1D ("Griffin：将门控线性循环与局部注意力混合以实现高效的
// 语言模型", §循环块: a small separable Conv1D with temporal filter width 4 ahead of the
// RG-LRU). u_t[c] = conv_b[c] + Σ_k conv_w[k][c] · x_{t-3+k}[c], zero history unless a
// conv state is given.
//
// Prefill: each thread owns 16 bytes of channels of one batch row and walks a run of
// kConvRun time steps with the three previous inputs held in registers, so x is read
// once (plus a 3-row halo per run) and u written once, both coalesced 16-byte accesses.
//
// Decode: one thread per 8 channels of one row; reads x_t and the 3-slot ring, writes u_t
// twice — rounded to bf16 as the gate GEMM's operand, and in float32 for the RG-LRU
// update in the GEMM epilogue (the same split as the prefill path, where the scan
// recomputes u in float32) — and overwrites the oldest ring slot with x_t. It also writes
// c·log σ(Λ) per channel, which the decode GEMM epilogue reads.
#include <cstdint>
#include <cuda_bf16.h>

#include "gate_math.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace rglru {
namespace {

constexpr int kConvThreads = 128;
constexpr int kConvRun = 32;

template <typename T> struct CV;
template <> struct CV<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void unpack(const uint4& v, float (&f)[8]) {
    f[0] = bf16lo(v.x); f[1] = bf16hi(v.x); f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
    f[4] = bf16lo(v.z); f[5] = bf16hi(v.z); f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
  }
  __device__ static uint4 pack(const float (&f)[8]) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7]));
  }
};
template <> struct CV<float> {
  static constexpr int N = 4;
  __device__ static void unpack(const uint4& v, float (&f)[4]) {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y); f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
  }
  __device__ static uint4 pack(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
  }
};

template <typename T>
__global__ void __launch_bounds__(kConvThreads) conv1d_fwd_kernel(const float* __restrict__ conv_w,
                                                                 const float* __restrict__ conv_b,
                                                                 const T* __restrict__ x, const T* __restrict__ state0,
                                                                 T* __restrict__ u, T* __restrict__ stateT, int B,
                                                                 int T_, int R) {
  constexpr int V = CV<T>::N;
  const int grp = blockIdx.x * kConvThreads + threadIdx.x;
  const int c0 = grp * V;
  if (c0 >= R) return;
  const int b = blockIdx.z;
  const int t0 = blockIdx.y * kConvRun;
  const int t1 = min(t0 + kConvRun, T_);

  float w[4][V], cb[V];
#pragma unroll
  for (int v = 0; v < V; ++v) {
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k][v] = __ldg(conv_w + k * R + c0 + v);
    cb[v] = __ldg(conv_b + c0 + v);
  }
  float hist[3][V];
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    const int t = t0 - 3 + j;
    uint4 raw = make_uint4(0, 0, 0, 0);
    if (t >= 0) raw = __ldg(reinterpret_cast<const uint4*>(x + ((int64_t)b * T_ + t) * R + c0));
    else if (state0 != nullptr)
      raw = __ldg(reinterpret_cast<const uint4*>(state0 + ((int64_t)b * 3 + (t + 3)) * R + c0));
    CV<T>::unpack(raw, hist[j]);
  }
  const T* xp = x + ((int64_t)b * T_) * R + c0;
  T* up = u + ((int64_t)b * T_) * R + c0;
  constexpr int U = 8;
  for (int t = t0; t < t1; t += U) {
    uint4 raw[U];
#pragma unroll
    for (int k = 0; k < U; ++k)
      if (t + k < t1) raw[k] = __ldcs(reinterpret_cast<const uint4*>(xp + (int64_t)(t + k) * R));
#pragma unroll
    for (int k = 0; k < U; ++k) {
      if (t + k < t1) {
        float xc[V], o[V];
        CV<T>::unpack(raw[k], xc);
#pragma unroll
        for (int v = 0; v < V; ++v) {
          float acc = cb[v];
          acc = fmaf(w[0][v], hist[0][v], acc);
          acc = fmaf(w[1][v], hist[1][v], acc);
          acc = fmaf(w[2][v], hist[2][v], acc);
          acc = fmaf(w[3][v], xc[v], acc);
          o[v] = acc;
          hist[0][v] = hist[1][v];
          hist[1][v] = hist[2][v];
          hist[2][v] = xc[v];
        }
        *reinterpret_cast<uint4*>(up + (int64_t)(t + k) * R) = CV<T>::pack(o);
      }
    }
  }
  if (stateT != nullptr && t1 == T_) {
#pragma unroll
    for (int j = 0; j < 3; ++j)
      *reinterpret_cast<uint4*>(stateT + ((int64_t)b * 3 + j) * R + c0) = CV<T>::pack(hist[j]);
  }
}

__global__ void __launch_bounds__(kConvThreads) decode_conv_kernel(const float* __restrict__ conv_w,
                                                                  const float* __restrict__ conv_b,
                                                                  const float* __restrict__ Lambda,
                                                                  const __nv_bfloat16* __restrict__ x_t,
                                                                  __nv_bfloat16* __restrict__ ring, int s0,
                                                                  __nv_bfloat16* __restrict__ u_t,
                                                                  float* __restrict__ u_f32,
                                                                  float* __restrict__ cla, unsigned* status, int B,
                                                                  int R) {
  constexpr int V = 8;
  const int c0 = (blockIdx.x * kConvThreads + threadIdx.x) * V;
  const int b = blockIdx.y;
  if (blockIdx.x == 0 && b == 0 && threadIdx.x == 0) *status = 0u;
  if (c0 >= R) return;
  const int s1 = (s0 + 1) % 3, s2 = (s0 + 2) % 3;
  float xo[V], xm2[V], xm1[V], xc[V], o[V];
  const uint4 raw_c = __ldcs(reinterpret_cast<const uint4*>(x_t + (int64_t)b * R + c0));
  __nv_bfloat16* rb = ring + (int64_t)b * 3 * R + c0;
  CV<__nv_bfloat16>::unpack(*reinterpret_cast<const uint4*>(rb + (int64_t)s0 * R), xo);
  CV<__nv_bfloat16>::unpack(*reinterpret_cast<const uint4*>(rb + (int64_t)s1 * R), xm2);
  CV<__nv_bfloat16>::unpack(*reinterpret_cast<const uint4*>(rb + (int64_t)s2 * R), xm1);
  CV<__nv_bfloat16>::unpack(raw_c, xc);
#pragma unroll
  for (int v = 0; v < V; ++v) {
    float acc = __ldg(conv_b + c0 + v);
    acc = fmaf(__ldg(conv_w + c0 + v), xo[v], acc);
    acc = fmaf(__ldg(conv_w + R + c0 + v), xm2[v], acc);
    acc = fmaf(__ldg(conv_w + 2 * R + c0 + v), xm1[v], acc);
    acc = fmaf(__ldg(conv_w + 3 * R + c0 + v), xc[v], acc);
    o[v] = acc;
  }
  *reinterpret_cast<uint4*>(u_t + (int64_t)b * R + c0) = CV<__nv_bfloat16>::pack(o);
  float4* uf = reinterpret_cast<float4*>(u_f32 + (int64_t)b * R + c0);
  uf[0] = make_float4(o[0], o[1], o[2], o[3]);
  uf[1] = make_float4(o[4], o[5], o[6], o[7]);
  *reinterpret_cast<uint4*>(rb + (int64_t)s0 * R) = raw_c;
  if (b == 0) {
#pragma unroll
    for (int v = 0; v < V; ++v) cla[c0 + v] = decay_log_coeff(__ldg(Lambda + c0 + v));
  }
}

}  // namespace

cudaError_t launch_conv1d(const float* conv_w, const float* conv_b, const void* x, const void* state0, void* u,
                          void* stateT, int B, int T, int R, bool bf16, cudaStream_t s) {
  const int V = bf16 ? 8 : 4;
  const int groups = R / V;
  dim3 grid((groups + kConvThreads - 1) / kConvThreads, (T + kConvRun - 1) / kConvRun, B);
  if (bf16)
    conv1d_fwd_kernel<__nv_bfloat16><<<grid, kConvThreads, 0, s>>>(
        conv_w, conv_b, static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(state0),
        static_cast<__nv_bfloat16*>(u), static_cast<__nv_bfloat16*>(stateT), B, T, R);
  else
    conv1d_fwd_kernel<float><<<grid, kConvThreads, 0, s>>>(conv_w, conv_b, static_cast<const float*>(x),
                                                           static_cast<const float*>(state0),
                                                           static_cast<float*>(u), static_cast<float*>(stateT), B,
                                                           T, R);
  return cudaGetLastError();
}

cudaError_t launch_decode_conv(const float* conv_w, const float* conv_b, const float* Lambda, const void* x_t,
                               void* ring, int64_t step, void* u_t, float* u_f32, float* cla, unsigned* status,
                               int B, int R, cudaStream_t s) {
  dim3 grid((R / 8 + kConvThreads - 1) / kConvThreads, B);
  const int s0 = (int)(step % 3);
  decode_conv_kernel<<<grid, kConvThreads, 0, s>>>(conv_w, conv_b, Lambda,
                                                   static_cast<const __nv_bfloat16*>(x_t),
                                                   static_cast<__nv_bfloat16*>(ring), s0,
                                                   static_cast<__nv_bfloat16*>(u_t), u_f32, cla, status, B, R);
  return cudaGetLastError();
}

}  // namespace rglru
