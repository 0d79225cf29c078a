// The elementwise kernels of the Hawk residual layer ("Griffin：将门控线性循环与局部注意力
// 混合以实现高效的语言模型", §残块 (residual block, Fig. 2(a)) and §MLP块 (gated MLP,
// Fig. 2(b))). The layer is
//     y = x + RecurrentBlock(RMSNorm₁(x)),   out = y + MLP(RMSNorm₂(y)),
//     MLP(n) = (GeLU(n W_gateᵀ) ⊙ n W_upᵀ) W_downᵀ;
// its linears run on the tcgen05 GEMM and the recurrent block on the RG-LRU kernels.
// What is left is HBM-bound and lives here:
//   * add_rmsnorm_kernel: the residual add y = x + o (rounded to bf16 once, as the
//     residual stream is stored) fused with the RMSNorm of y that the next component
//     reads, n = y / √(mean y² + ε) ⊙ γ; either half may be skipped. One warp per row
//     of D channels, 16-byte loads and stores.
//   * gelu_mul_kernel: p = GeLU(gate) ⊙ up, exact erf GeLU, written over gate.
#include <algorithm>
#include <cstdint>
#include <cuda_bf16.h>

#include "gate_math.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace rglru {
namespace {

constexpr int kNormRowsPerBlock = 8;  // one warp per row
constexpr int kEwThreads = 256;

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  f[0] = bf16lo(v.x); f[1] = bf16hi(v.x); f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
  f[4] = bf16lo(v.z); f[5] = bf16hi(v.z); f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

// rows × D bf16 (D8 = D/8 vectors of 8 per row). o == nullptr: no add, the norm reads x.
// n == nullptr: no norm. x, o, y, n are distinct buffers.
__global__ void __launch_bounds__(kNormRowsPerBlock * 32)
add_rmsnorm_kernel(const uint4* __restrict__ x, const uint4* __restrict__ o, uint4* __restrict__ y,
                   uint4* __restrict__ n, const float4* __restrict__ scale, int64_t rows, int D8, float eps) {
  const int64_t row = (int64_t)blockIdx.x * kNormRowsPerBlock + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int64_t base = row * D8;
  float ss = 0.0f;
  for (int j = lane; j < D8; j += 32) {
    uint4 v = x[base + j];
    if (o != nullptr) {
      float a[8], b[8];
      unpack8(v, a);
      unpack8(o[base + j], b);
#pragma unroll
      for (int k = 0; k < 8; ++k) a[k] += b[k];
      v = pack8(a);
      y[base + j] = v;
    }
    if (n != nullptr) {
      float a[8];
      unpack8(v, a);
#pragma unroll
      for (int k = 0; k < 8; ++k) ss = fmaf(a[k], a[k], ss);
    }
  }
  if (n == nullptr) return;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  const float rstd = 1.0f / sqrtf(ss / (float)(D8 * 8) + eps);
  for (int j = lane; j < D8; j += 32) {
    float a[8];
    unpack8(o != nullptr ? y[base + j] : x[base + j], a);  // y: this thread's own stores above
    const float4 g0 = scale[2 * j], g1 = scale[2 * j + 1];
    a[0] *= rstd * g0.x; a[1] *= rstd * g0.y; a[2] *= rstd * g0.z; a[3] *= rstd * g0.w;
    a[4] *= rstd * g1.x; a[5] *= rstd * g1.y; a[6] *= rstd * g1.z; a[7] *= rstd * g1.w;
    n[base + j] = pack8(a);
  }
}

// n8 vectors of 8 bf16; p may be gate (in place: each vector is read before it is written).
__global__ void __launch_bounds__(kEwThreads)
gelu_mul_kernel(const uint4* gate, const uint4* __restrict__ up, uint4* p, int64_t n8) {
  const int64_t stride = (int64_t)gridDim.x * kEwThreads;
  for (int64_t i = (int64_t)blockIdx.x * kEwThreads + threadIdx.x; i < n8; i += stride) {
    float g[8], u[8];
    unpack8(gate[i], g);
    unpack8(up[i], u);
#pragma unroll
    for (int k = 0; k < 8; ++k) g[k] = gelu_exact(g[k]) * u[k];
    p[i] = pack8(g);
  }
}

}  // namespace

cudaError_t launch_add_rmsnorm(const void* x, const void* o, void* y, void* n, const float* scale, int64_t rows,
                               int D, float eps, cudaStream_t s) {
  if (rows < 1 || D < 8 || D % 8 != 0 || x == nullptr || (o != nullptr && y == nullptr) ||
      (n != nullptr && scale == nullptr) || (o == nullptr && n == nullptr))
    return cudaErrorInvalidValue;
  const int64_t blocks = (rows + kNormRowsPerBlock - 1) / kNormRowsPerBlock;
  if (blocks > INT32_MAX) return cudaErrorInvalidValue;
  add_rmsnorm_kernel<<<(unsigned)blocks, kNormRowsPerBlock * 32, 0, s>>>(
      static_cast<const uint4*>(x), static_cast<const uint4*>(o), static_cast<uint4*>(y), static_cast<uint4*>(n),
      reinterpret_cast<const float4*>(scale), rows, D / 8, eps);
  return cudaGetLastError();
}

cudaError_t launch_gelu_mul(const void* gate, const void* up, void* p, int64_t n, cudaStream_t s) {
  if (n < 8 || n % 8 != 0 || gate == nullptr || up == nullptr || p == nullptr) return cudaErrorInvalidValue;
  const int64_t n8 = n / 8;
  const int64_t want = (n8 + kEwThreads - 1) / kEwThreads;
  const int grid = (int)std::min<int64_t>(want, (int64_t)std::max(1, num_sms()) * 8);
  gelu_mul_kernel<<<grid, kEwThreads, 0, s>>>(static_cast<const uint4*>(gate), static_cast<const uint4*>(up),
                                              static_cast<uint4*>(p), n8);
  return cudaGetLastError();
}

}  // namespace rglru
