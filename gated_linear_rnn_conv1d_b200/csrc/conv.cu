// Width-4 causal depthwise Conv1D ("Griffin：将门控线性循环与局部注意力混合以实现高效的
// 语言模型", §循环块: a small separable Conv1D with temporal filter width 4 ahead of the
// RG-LRU). u_t[c] = conv_b[c] + Σ_k conv_w[k][c] · x_{t-3+k}[c], zero history unless a
// conv state is given.
//
// Prefill: tiles of one batch row × 128 (bf16) or 64 (f32) channels × 64 steps; x arrives
// in shared memory by one TMA copy including the 3-row halo, and each thread writes 4
// steps of 16 bytes of channels of u with coalesced stores.
//
// Decode: one thread per 8 channels of one row; reads x_t and the 3-slot ring, writes u_t
// twice — rounded to bf16 as the gate GEMM's operand, and in float32 for the RG-LRU
// update in the GEMM epilogue (the same split as the prefill path, where the scan
// recomputes u in float32) — and overwrites the oldest ring slot with x_t. It also writes
// c·log σ(Λ) per channel, which the decode GEMM epilogue reads.
#include <algorithm>
#include <cstdint>
#include <cuda_bf16.h>

#include "gate_math.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace rglru {
namespace {

constexpr int kConvThreads = 128;

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

// Prefill: persistent CTAs stream tiles of one batch row × CW channels (16 bytes per
// thread × 16 threads) × 64 steps through a ring of kConvStages shared-memory stages. One
// thread keeps kConvStages TMA copies in flight (each brings the tile's 67 x rows, the
// 3-row halo included; rows before t = 0 and channels past R arrive as zeros); the 256
// threads each produce 4 steps × V channels of u per tile.
constexpr int kTileThreads = 256;
constexpr int kTileSteps = 64;
constexpr int kTileRows = kTileSteps + 3;
constexpr int kConvStages = 4;

__device__ __forceinline__ void tma_load_x3(void* dst, const CUtensorMap* m, uint64_t* bar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Each CTA keeps one channel block (cblk = blockIdx.x mod n_cblk) for its whole life, so
// its taps and bias are loaded once; it walks that block's (batch row, time chunk) tiles.
template <typename T>
__global__ void __launch_bounds__(kTileThreads) conv1d_tile_kernel(const __grid_constant__ CUtensorMap mx,
                                                                  const float* __restrict__ conv_w,
                                                                  const float* __restrict__ conv_b,
                                                                  const T* __restrict__ state0, T* __restrict__ u,
                                                                  T* __restrict__ stateT, int B, int T_, int R,
                                                                  int n_cblk, int n_chunks, unsigned* status,
                                                                  uint4* __restrict__ zero, int64_t zero_n16) {
  constexpr int V = CV<T>::N;
  constexpr int CW = 16 * V;
  constexpr int kStage = kTileRows * CW * (int)sizeof(T);
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* sbase = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  __shared__ __align__(8) uint64_t full[kConvStages];

  const int tid = threadIdx.x;
  // the next kernel (launched as a programmatic dependent) may be scheduled from now on
  pdl_launch_dependents();
  // zero the scan's workspace header and carries for the kernels after this one (saves a
  // separate memset launch); its status word is set only after a wait of about a second,
  // long after every CTA of this grid has passed this point
  for (int64_t i = (int64_t)blockIdx.x * kTileThreads + tid; i < zero_n16; i += (int64_t)gridDim.x * kTileThreads)
    zero[i] = make_uint4(0u, 0u, 0u, 0u);
  const int g = tid % 16, s = tid / 16;
  const int cblk = blockIdx.x % n_cblk;
  const int lane0 = blockIdx.x / n_cblk;         // first (b, chunk) pair of this CTA
  const int stride = gridDim.x / n_cblk;         // CTAs sharing this channel block
  const int n_pairs = B * n_chunks;
  auto issue = [&](int k, int pair) {
    const int b = pair / n_chunks, chunk = pair % n_chunks;
    mbar_arrive_expect_tx(&full[k], kStage);
    tma_load_x3(sbase + k * kStage, &mx, &full[k], cblk * CW, chunk * kTileSteps - 3, b);
  };
  if (tid == 0) {
    for (int k = 0; k < kConvStages; ++k) mbar_init(&full[k], 1);
    fence_barrier_init();
    for (int k = 0; k < kConvStages; ++k) {
      const int pair = lane0 + k * stride;
      if (pair < n_pairs) issue(k, pair);
    }
  }
  const int c0 = cblk * CW + g * V;
  const bool cvalid = c0 < R;
  float w[4][V], cb[V];
#pragma unroll
  for (int v = 0; v < V; v += 4) {
    const int c = cvalid ? c0 + v : 0;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(conv_w + kk * R + c));
      w[kk][v] = f.x; w[kk][v + 1] = f.y; w[kk][v + 2] = f.z; w[kk][v + 3] = f.w;
    }
    const float4 f = __ldg(reinterpret_cast<const float4*>(conv_b + c));
    cb[v] = f.x; cb[v + 1] = f.y; cb[v + 2] = f.z; cb[v + 3] = f.w;
  }
  __syncthreads();
  volatile int no_abort = 0;
  int it = 0;
  for (int pair = lane0; pair < n_pairs; pair += stride, ++it) {
    const int k = it % kConvStages;
    const uint32_t parity = (uint32_t)((it / kConvStages) & 1);
    T* sx = reinterpret_cast<T*>(sbase + k * kStage);
    const int b = pair / n_chunks, chunk = pair % n_chunks;
    const int t0 = chunk * kTileSteps;
    if (!mbar_wait(&full[k], parity, &no_abort) && tid == 0) atomicOr(status, kStatusTimeout);
    if (chunk == 0 && state0 != nullptr) {
      __syncthreads();
      if (tid < 48) {
        // conv history before t = 0 comes from the given state instead of zeros
        const int j = tid / 16, gg = tid % 16, cc = cblk * CW + gg * V;
        if (cc < R)
          *reinterpret_cast<uint4*>(sx + j * CW + gg * V) =
              __ldg(reinterpret_cast<const uint4*>(state0 + ((int64_t)b * 3 + j) * R + cc));
      }
      __syncthreads();
    }
    if (cvalid) {
      float hist[3][V];
#pragma unroll
      for (int j = 0; j < 3; ++j) CV<T>::unpack(*reinterpret_cast<const uint4*>(sx + (s * 4 + j) * CW + g * V), hist[j]);
#pragma unroll
      for (int l = 0; l < 4; ++l) {
        const int t = t0 + s * 4 + l;
        float xc[V], o[V];
        CV<T>::unpack(*reinterpret_cast<const uint4*>(sx + (s * 4 + l + 3) * CW + g * V), xc);
#pragma unroll
        for (int v = 0; v < V; v += 2) {
          float2 a2 = __ffma2_rn(make_float2(w[0][v], w[0][v + 1]), make_float2(hist[0][v], hist[0][v + 1]),
                                 make_float2(cb[v], cb[v + 1]));
          a2 = __ffma2_rn(make_float2(w[1][v], w[1][v + 1]), make_float2(hist[1][v], hist[1][v + 1]), a2);
          a2 = __ffma2_rn(make_float2(w[2][v], w[2][v + 1]), make_float2(hist[2][v], hist[2][v + 1]), a2);
          a2 = __ffma2_rn(make_float2(w[3][v], w[3][v + 1]), make_float2(xc[v], xc[v + 1]), a2);
          o[v] = a2.x;
          o[v + 1] = a2.y;
        }
#pragma unroll
        for (int v = 0; v < V; ++v) {
          hist[0][v] = hist[1][v];
          hist[1][v] = hist[2][v];
          hist[2][v] = xc[v];
        }
        if (t < T_) __stcg(reinterpret_cast<uint4*>(u + ((int64_t)b * T_ + t) * R + c0), CV<T>::pack(o));
      }
    }
    if (stateT != nullptr && chunk == n_chunks - 1 && tid < 48) {
      // the last three inputs x_{T-3}, x_{T-2}, x_{T-1} sit at tile rows T − t0 … T − t0 + 2
      const int j = tid / 16, gg = tid % 16, cc = cblk * CW + gg * V;
      if (cc < R)
        *reinterpret_cast<uint4*>(stateT + ((int64_t)b * 3 + j) * R + cc) =
            *reinterpret_cast<const uint4*>(sx + (T_ - t0 + j) * CW + gg * V);
    }
    __syncthreads();  // stage k fully read
    if (tid == 0) {
      const int np = pair + kConvStages * stride;
      if (np < n_pairs) issue(k, np);
    }
  }
}

// 8 consecutive floats (16-byte aligned) through the read-only path
__device__ __forceinline__ void ld8(const float* p, float (&f)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
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
  // the step GEMM that follows may start its prologue now; it waits for this grid's results
  pdl_launch_dependents();
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
  // taps and bias of the thread's 8 channels as 16-byte loads (parameters are 16-byte
  // aligned, c0 a multiple of 8 and R of 8)
  float w0[V], w1[V], w2[V], w3[V], cb[V];
  ld8(conv_w + c0, w0);
  ld8(conv_w + R + c0, w1);
  ld8(conv_w + 2 * R + c0, w2);
  ld8(conv_w + 3 * R + c0, w3);
  ld8(conv_b + c0, cb);
#pragma unroll
  for (int v = 0; v < V; ++v) {
    float acc = cb[v];
    acc = fmaf(w0[v], xo[v], acc);
    acc = fmaf(w1[v], xm2[v], acc);
    acc = fmaf(w2[v], xm1[v], acc);
    acc = fmaf(w3[v], xc[v], acc);
    o[v] = acc;
  }
  *reinterpret_cast<uint4*>(u_t + (int64_t)b * R + c0) = CV<__nv_bfloat16>::pack(o);
  float4* uf = reinterpret_cast<float4*>(u_f32 + (int64_t)b * R + c0);
  uf[0] = make_float4(o[0], o[1], o[2], o[3]);
  uf[1] = make_float4(o[4], o[5], o[6], o[7]);
  *reinterpret_cast<uint4*>(rb + (int64_t)s0 * R) = raw_c;
  if (b == 0) {
    float lam[V];
    ld8(Lambda + c0, lam);
#pragma unroll
    for (int v = 0; v < V; ++v) lam[v] = decay_log_coeff(lam[v]);
    float4* cp = reinterpret_cast<float4*>(cla + c0);
    cp[0] = make_float4(lam[0], lam[1], lam[2], lam[3]);
    cp[1] = make_float4(lam[4], lam[5], lam[6], lam[7]);
  }
}

}  // namespace

cudaError_t launch_conv1d(const float* conv_w, const float* conv_b, const void* x, const void* state0, void* u,
                          void* stateT, int B, int T, int R, bool bf16, unsigned* status, cudaStream_t s, void* zero,
                          size_t zero_bytes) {
  if (zero_bytes % 16 != 0 || (zero_bytes != 0 && (reinterpret_cast<uintptr_t>(zero) & 15) != 0))
    return cudaErrorInvalidValue;
  const int es = bf16 ? 2 : 4;
  const int cw = bf16 ? 128 : 64;
  const int n_cblk = (R + cw - 1) / cw;
  const int n_chunks = (T + kTileSteps - 1) / kTileSteps;
  const int64_t tiles = (int64_t)B * n_cblk * n_chunks;
  if (tiles > INT32_MAX) return cudaErrorInvalidValue;
  EncodeTiledFn fn = get_encode_tiled();
  if (fn == nullptr) return cudaErrorInvalidValue;
  CUtensorMap mx;
  cuuint64_t dims[3] = {(cuuint64_t)R, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[2] = {(cuuint64_t)R * es, (cuuint64_t)T * R * es};
  cuuint32_t box[3] = {(cuuint32_t)cw, (cuuint32_t)kTileRows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  if (fn(&mx, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(x), dims,
         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const int smem = kConvStages * kTileRows * cw * es + 128;
  static bool attr[2][64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr[bf16][dev]) {
    e = bf16 ? cudaFuncSetAttribute(conv1d_tile_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)
             : cudaFuncSetAttribute(conv1d_tile_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr[bf16][dev] = true;
  }
  // a multiple of n_cblk CTAs, about two per SM; each keeps one channel block
  const int64_t pairs = (int64_t)B * n_chunks;
  int64_t per_blk = std::max<int64_t>(1, (int64_t)2 * num_sms() / n_cblk);
  per_blk = std::min<int64_t>(per_blk, pairs);
  const int64_t grid = per_blk * n_cblk;
  if (grid > INT32_MAX) return cudaErrorInvalidValue;
  if (bf16)
    conv1d_tile_kernel<__nv_bfloat16><<<(unsigned)grid, kTileThreads, smem, s>>>(
        mx, conv_w, conv_b, static_cast<const __nv_bfloat16*>(state0), static_cast<__nv_bfloat16*>(u),
        static_cast<__nv_bfloat16*>(stateT), B, T, R, n_cblk, n_chunks, status, static_cast<uint4*>(zero),
        (int64_t)(zero_bytes / 16));
  else
    conv1d_tile_kernel<float><<<(unsigned)grid, kTileThreads, smem, s>>>(
        mx, conv_w, conv_b, static_cast<const float*>(state0), static_cast<float*>(u), static_cast<float*>(stateT), B,
        T, R, n_cblk, n_chunks, status, static_cast<uint4*>(zero), (int64_t)(zero_bytes / 16));
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
