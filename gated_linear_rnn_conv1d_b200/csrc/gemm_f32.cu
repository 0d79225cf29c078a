// float32 gate projections for the float32-IO path: z = u [W_a | W_x]ᵀ + [b_a | b_x]
// ("Griffin：将门控线性循环与局部注意力混合以实现高效的语言模型", §实门线性循环单元
// (RG-LRU), Eq. (1)–(2) arguments of σ), FFMA on the CUDA cores so that the result keeps
// float32 accuracy (no TF32 rounding). Output in the packed gate layout: column
// 256·(c/128) + (c%128) holds channel c's z_a, the same column + 128 its z_x.
//
// Classic register-tiled SIMT GEMM: a 64×64 output tile per 256-thread CTA, each thread a
// 4×4 sub-tile, K staged through shared memory 16 at a time.
#include <cstdint>

#include "kernels.cuh"

namespace rglru {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

__global__ void __launch_bounds__(256) gemm_gates_f32_kernel(const float* __restrict__ u, const float* __restrict__ Wa,
                                                            const float* __restrict__ ba, const float* __restrict__ Wx,
                                                            const float* __restrict__ bx, float* __restrict__ z,
                                                            int64_t M, int R, int64_t pitch) {
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int64_t m0 = (int64_t)blockIdx.y * TM;
  const int n0 = blockIdx.x * TN;  // packed column

  // packed column n → (weight matrix, channel)
  auto wrow = [&](int n, int& ch) -> const float* {
    const int blk = n / 256, w = n % 256;
    ch = blk * 128 + (w % 128);
    return (w < 128) ? Wa : Wx;
  };

  float acc[4][4] = {};
  for (int k0 = 0; k0 < R; k0 += TK) {
    // load A tile: 64 rows × 16 k (256 threads × 4 elements)
    for (int i = threadIdx.x; i < TM * TK; i += 256) {
      const int r = i / TK, k = i % TK;
      const int64_t m = m0 + r;
      As[k][r] = (m < M && k0 + k < R) ? u[m * R + k0 + k] : 0.0f;
    }
    for (int i = threadIdx.x; i < TN * TK; i += 256) {
      const int c = i / TK, k = i % TK;
      int ch;
      const float* W = wrow(n0 + c, ch);
      Bs[k][c] = (ch < R && k0 + k < R) ? W[(int64_t)ch * R + k0 + k] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < TK; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[k][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[k][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      const int blk = n / 256, w = n % 256;
      const int ch = blk * 128 + (w % 128);
      if (n < pitch && ch < R) z[m * pitch + n] = acc[i][j] + ((w < 128) ? ba[ch] : bx[ch]);
    }
  }
}

}  // namespace

cudaError_t launch_gemm_gates_f32(const float* u, const float* Wa, const float* ba, const float* Wx,
                                  const float* bx, float* z, int64_t M, int R, cudaStream_t s) {
  const int64_t pitch = gate_pitch(R);
  dim3 grid((unsigned)((pitch + TN - 1) / TN), (unsigned)((M + TM - 1) / TM));
  gemm_gates_f32_kernel<<<grid, 256, 0, s>>>(u, Wa, ba, Wx, bx, z, M, R, pitch);
  return cudaGetLastError();
}

}  // namespace rglru
