// float32 gate projections for the float32-IO path: z = u [W_a | W_x]ᵀ + [b_a | b_x]
// ("Griffin：将门控线性循环与局部注意力混合以实现高效的语言模型", §实门线性循环单元
// (RG-LRU), Eq. (1)–(2) arguments of σ), FFMA on the CUDA cores so that the result keeps
// float32 accuracy (no TF32 rounding). Output in the packed gate layout: column
// 256·(c/128) + (c%128) holds channel c's z_a, the same column + 128 its z_x.
//
// Register-tiled SIMT GEMM: a TM×TN output tile per 256-thread CTA (16×16 threads, each a
// (TM/16)×(TN/16) sub-tile), K staged through shared memory 32 at a time in two buffers, the
// next K tile's loads issued into registers before the current one is multiplied. 64×64
// tiles when they fill the GPU twice over, 32×32 otherwise (small problems are latency-bound:
// one float32 decode-size gate projection is 32 CTAs of 64×64 on a 148-SM part).
#include <cstdint>

#include "kernels.cuh"
#include "ptx.cuh"

namespace rglru {
namespace {

constexpr int TK = 32;

template <int TM, int TN>
__global__ void __launch_bounds__(256) gemm_gates_f32_kernel(const float* __restrict__ u, const float* __restrict__ Wa,
                                                            const float* __restrict__ ba, const float* __restrict__ Wx,
                                                            const float* __restrict__ bx, float* __restrict__ z,
                                                            int64_t M, int R, int64_t pitch) {
  // launched as a programmatic dependent: u is the previous kernel's (the Conv1D's) output
  pdl_wait();
  pdl_launch_dependents();
  constexpr int RM = TM / 16, RN = TN / 16;           // per-thread sub-tile
  constexpr int LA = TM * TK / 256, LB = TN * TK / 256;  // loads per thread per K tile
  __shared__ float As[2][TK][TM + 4];
  __shared__ float Bs[2][TK][TN + 4];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int64_t m0 = (int64_t)blockIdx.y * TM;
  const int n0 = blockIdx.x * TN;  // packed column

  // packed column n → (weight matrix, channel)
  auto wrow = [&](int n, int& ch) -> const float* {
    const int blk = n / 256, w = n % 256;
    ch = blk * 128 + (w % 128);
    return (w < 128) ? Wa : Wx;
  };
  // element i of this thread's share of a K tile: (row or column, k) with k fastest, so that
  // 32 consecutive threads read 32 consecutive floats of one row
  float ra[LA], rb[LB];
  auto load = [&](int k0) {
#pragma unroll
    for (int q = 0; q < LA; ++q) {
      const int i = threadIdx.x + q * 256, r = i / TK, k = i % TK;
      const int64_t m = m0 + r;
      ra[q] = (m < M && k0 + k < R) ? u[m * R + k0 + k] : 0.0f;
    }
#pragma unroll
    for (int q = 0; q < LB; ++q) {
      const int i = threadIdx.x + q * 256, c = i / TK, k = i % TK;
      int ch;
      const float* W = wrow(n0 + c, ch);
      rb[q] = (ch < R && k0 + k < R) ? W[(int64_t)ch * R + k0 + k] : 0.0f;
    }
  };
  auto store = [&](int buf) {
#pragma unroll
    for (int q = 0; q < LA; ++q) {
      const int i = threadIdx.x + q * 256;
      As[buf][i % TK][i / TK] = ra[q];
    }
#pragma unroll
    for (int q = 0; q < LB; ++q) {
      const int i = threadIdx.x + q * 256;
      Bs[buf][i % TK][i / TK] = rb[q];
    }
  };

  float acc[RM][RN] = {};
  load(0);
  store(0);
  __syncthreads();
  int buf = 0;
  for (int k0 = 0; k0 < R; k0 += TK) {
    const bool more = k0 + TK < R;
    if (more) load(k0 + TK);  // in flight while this tile is multiplied
#pragma unroll
    for (int k = 0; k < TK; ++k) {
      float a[RM], b[RN];
#pragma unroll
      for (int i = 0; i < RM; ++i) a[i] = As[buf][k][ty * RM + i];
#pragma unroll
      for (int j = 0; j < RN; ++j) b[j] = Bs[buf][k][tx * RN + j];
#pragma unroll
      for (int i = 0; i < RM; ++i)
#pragma unroll
        for (int j = 0; j < RN; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    if (more) {
      store(buf ^ 1);  // the other buffer: its last readers passed the barrier below
      __syncthreads();
      buf ^= 1;
    }
  }
#pragma unroll
  for (int i = 0; i < RM; ++i) {
    const int64_t m = m0 + ty * RM + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < RN; ++j) {
      const int n = n0 + tx * RN + j;
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
  const int64_t big = ((pitch + 63) / 64) * ((M + 63) / 64);
  // programmatic dependent launch: the CTAs start while the previous kernel finishes and
  // wait (griddepcontrol.wait) before reading its output
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (big >= 2 * num_sms()) {
    cfg.gridDim = dim3((unsigned)((pitch + 63) / 64), (unsigned)((M + 63) / 64));
    return cudaLaunchKernelEx(&cfg, gemm_gates_f32_kernel<64, 64>, u, Wa, ba, Wx, bx, z, M, R, pitch);
  }
  cfg.gridDim = dim3((unsigned)((pitch + 31) / 32), (unsigned)((M + 31) / 32));
  return cudaLaunchKernelEx(&cfg, gemm_gates_f32_kernel<32, 32>, u, Wa, ba, Wx, bx, z, M, R, pitch);
}

}  // namespace rglru
