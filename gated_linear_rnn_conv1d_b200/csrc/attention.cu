// Decode step of Griffin's local multi-query attention on the sm_100a tensor cores.
//
// "Griffin：将门控线性循环与局部注意力混合以实现高效的语言模型", §时间混合块: MQA (H query
// heads of D_head = 128, H·D_head = D, one key/value head shared by all of them), RoPE as
// the relative position embedding, local sliding-window attention (each position sees a
// fixed number of past positions, which bounds the KV cache by the window); "Griffin's
// Compromise: Combining Gated Linear Recurrence with Local Attention", §Griffin: window
// 1024.
//
// One step at position `pos` for B sequences:
//   attn_prep_kernel   from the fused projection qkv = x W_qkvᵀ: rotates q and k (RoPE,
//                      pair i = (x_{2i}, x_{2i+1}) turned by pos·θ_i, θ_i = 10000^(−2i/128),
//                      the angle reduced in float64), writes the rotated queries, the key
//                      into slot (pos mod W) of the key ring and the value into the same
//                      slot of the (transposed) value ring;
//   attn_chunk_kernel  one CTA per (sequence, 128-slot chunk of the ring): TMA brings the
//                      chunk's keys [128 slots][128], values [128 dims][128 slots] and the
//                      sequence's queries [H][128] into 128-byte-swizzled shared memory;
//                      tcgen05.mma forms Sᵀ = K·Qᵀ (M = 128 slots, N = H heads, fp32 in
//                      TMEM); the four warps turn it into this chunk's softmax numerators
//                      P = 2^(s − m) (bf16, written in the swizzled layout the tensor core
//                      reads) with the chunk's per-head maximum m and sum l; a second MMA
//                      forms Oᵀ = Vᵀ·Pᵀ (M = 128 dims, N = H); the partial output, m and l
//                      go to the workspace. Slots not yet written (pos < W − 1) are masked.
//   attn_combine_kernel  merges the chunks of each sequence and head (flash-decoding):
//                      o = Σ_c 2^(m_c − m*) O_c / Σ_c 2^(m_c − m*) l_c, in bf16.
// The q, k, v and output projections run on the tcgen05 GEMM of gemm_tc.cu.
//
// Ring layouts: keys [B][W][128] (slot-major), values [B][128][W] (dimension-major, so that
// Vᵀ is a K-major operand like every other one: no transposed descriptor is needed). The
// attention is a sum over the window's slots, so they are read in slot order whatever
// position each holds. Every wait is bounded.
#include <cmath>
#include <cstdint>
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace rglru {
namespace {

constexpr int kDh = 128;          // D_head
constexpr int kChunk = 128;       // ring slots per CTA
constexpr int kAttnThreads = 128;
constexpr float kLog2e = 1.4426950408889634f;

struct AttnSmem {
  // offsets from the 1024-aligned base; every TMA box and operand tile starts 1024-aligned
  int hp;                       // heads rounded up to 16 (the MMA's N)
  int off_k, off_v, off_q, off_p, off_s, bytes;
};
__host__ __device__ inline AttnSmem attn_smem(int H) {
  AttnSmem L;
  L.hp = (H + 15) / 16 * 16;
  L.off_k = 0;                                   // 2 boxes [128 slots][64 dims]
  L.off_v = L.off_k + 2 * kChunk * 128;          // 2 boxes [128 dims][64 slots]
  L.off_q = L.off_v + 2 * kDh * 128;             // 2 boxes [hp heads][64 dims]
  L.off_p = L.off_q + ((2 * L.hp * 128 + 1023) / 1024) * 1024;  // 2 k-blocks [hp][64 slots]
  L.off_s = L.off_p + ((2 * L.hp * 128 + 1023) / 1024) * 1024;  // scores [hp][128] float
  L.bytes = L.off_s + L.hp * kChunk * 4;
  return L;
}

struct AttnArgs {
  const __nv_bfloat16* qkv;  // [B][(H+2)·128]
  __nv_bfloat16* q_rot;      // [B][H][128]
  __nv_bfloat16* k_ring;     // [B][W][128]
  __nv_bfloat16* v_ring;     // [B][128][W]
  float* o_part;             // [B][n_chunks][H][128]
  float* m_part;             // [B][n_chunks][H]
  float* l_part;             // [B][n_chunks][H]
  __nv_bfloat16* o;          // [B][H·128]
  unsigned* status;
  int64_t pos;
  int B, H, W, n_chunks;
};

// ---- RoPE, ring writes --------------------------------------------------------------
__global__ void __launch_bounds__(256) attn_prep_kernel(AttnArgs a) {
  pdl_wait();  // qkv is the previous kernel's output
  pdl_launch_dependents();
  const int b = blockIdx.x;
  const int H = a.H;
  const int64_t nq = (int64_t)(H + 2) * kDh;
  const __nv_bfloat16* src = a.qkv + (int64_t)b * nq;
  const int slot = (int)(a.pos % a.W);
  // rotation pairs of the H query heads and the key: (H + 1) · 64 of them
  for (int i = threadIdx.x; i < (H + 1) * (kDh / 2); i += blockDim.x) {
    const int head = i / (kDh / 2), j = i % (kDh / 2);
    // θ_j = 10000^(−2j/128); the angle pos·θ_j reduced modulo 2π in float64, so that large
    // positions keep their accuracy
    const double theta = exp(-(double)j * (2.0 / kDh) * 9.210340371976184);  // ln 10000
    double ang = fmod((double)a.pos * theta, 6.283185307179586);
    double sd, cd;
    sincos(ang, &sd, &cd);
    const float s = (float)sd, c = (float)cd;
    const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(src + head * kDh + 2 * j);
    const float x0 = __bfloat162float(v.x), x1 = __bfloat162float(v.y);
    const __nv_bfloat162 r = __floats2bfloat162_rn(x0 * c - x1 * s, x0 * s + x1 * c);
    if (head < H)
      *reinterpret_cast<__nv_bfloat162*>(a.q_rot + ((int64_t)b * H + head) * kDh + 2 * j) = r;
    else
      *reinterpret_cast<__nv_bfloat162*>(a.k_ring + ((int64_t)b * a.W + slot) * kDh + 2 * j) = r;
  }
  // the value, unrotated, into the transposed ring
  for (int d = threadIdx.x; d < kDh; d += blockDim.x)
    a.v_ring[((int64_t)b * kDh + d) * a.W + slot] = src[(int64_t)(H + 1) * kDh + d];
}

// ---- one ring chunk of one sequence ------------------------------------------------------
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* m, uint64_t* bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// byte offset of element (row, k) of a K-major bf16 tile stored with the 128-byte swizzle:
// rows of 64 elements (128 bytes), 16-byte chunks permuted by (row mod 8)
__device__ __forceinline__ uint32_t sw128_offset(int row, int k) {
  return (uint32_t)row * 128u + ((uint32_t)((k >> 3) ^ (row & 7)) << 4) + (uint32_t)(k & 7) * 2u;
}

__global__ void __launch_bounds__(kAttnThreads, 2)
    attn_chunk_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmQ, AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t load_bar, mma1_bar, mma2_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const AttnSmem L = attn_smem(a.H);
  const int hp = L.hp;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int c = blockIdx.x, b = blockIdx.y;
  const int64_t part = (int64_t)b * a.n_chunks + c;
  // slots of this chunk that hold a position of the window: all once the ring has wrapped
  // (pos ≥ W − 1), otherwise slots 0 … pos
  const int64_t first = (int64_t)c * kChunk;
  const int n_valid = a.pos >= a.W - 1 ? kChunk : (int)max((int64_t)0, min((int64_t)kChunk, a.pos + 1 - first));

  pdl_wait();  // the ring and the rotated queries are the previous kernel's output
  pdl_launch_dependents();
  if (n_valid == 0) {
    for (int h = threadIdx.x; h < a.H; h += blockDim.x) {
      a.m_part[part * a.H + h] = -INFINITY;
      a.l_part[part * a.H + h] = 0.0f;
    }
    return;
  }
  if (threadIdx.x == 0) {
    mbar_init(&load_bar, 1);
    mbar_init(&mma1_bar, 1);
    mbar_init(&mma2_bar, 1);
    abort_s = 0;
    fence_barrier_init();
  }
  // Sᵀ in columns [0, hp), Oᵀ in [hp, 2hp); 32 more so that every 32-column load of the
  // last group stays inside the allocation
  const int need = 2 * hp + 32;
  const uint32_t tmem_cols = need <= 64 ? 64u : (need <= 128 ? 128u : (need <= 256 ? 256u : 512u));
  if (warp == 0) {
    tmem_alloc(&tmem_base_s, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  uint8_t* sK = smem + L.off_k;
  uint8_t* sV = smem + L.off_v;
  uint8_t* sQ = smem + L.off_q;
  uint8_t* sP = smem + L.off_p;
  float* sS = reinterpret_cast<float*>(smem + L.off_s);
  const uint32_t idesc = umma_idesc_bf16_f32(128, hp);
  static_assert(kAttnMaxHeads <= 128, "the N of both MMAs, and 2·N + 32 TMEM columns, stay in range");
  bool ok = true;

  if (threadIdx.x == 0) {
    const uint32_t bytes = 2 * kChunk * 128 + 2 * kDh * 128 + 2 * hp * 128;
    mbar_arrive_expect_tx(&load_bar, bytes);
    for (int kb = 0; kb < 2; ++kb) {
      tma_load_3d(sK + kb * kChunk * 128, &tmK, &load_bar, kb * 64, (int)first, b);  // keys, dims kb·64…
      tma_load_3d(sV + kb * kDh * 128, &tmV, &load_bar, (int)first + kb * 64, 0, b);  // values, slots …
      tma_load_3d(sQ + kb * hp * 128, &tmQ, &load_bar, kb * 64, 0, b);               // queries (rows ≥ H: 0)
    }
    if (!mbar_wait(&load_bar, 0, &abort_s)) ok = false;
    if (ok) {
      tc_fence_after();
      // Sᵀ[slot][head] = Σ_d K[slot][d] Q[head][d]
      for (int kb = 0; kb < 2; ++kb)
        for (int k = 0; k < 4; ++k)
          umma_f16(tmem, umma_desc_sw128(smem_u32(sK + kb * kChunk * 128) + k * 32),
                   umma_desc_sw128(smem_u32(sQ + kb * hp * 128) + k * 32), idesc, (kb | k) != 0 ? 1u : 0u);
      umma_commit(&mma1_bar);
    } else {
      abort_s = 1;
      atomicOr(a.status, kStatusTimeout);
    }
  }
  // scores → shared memory as sS[head][slot], scaled to log2 units; unwritten slots −inf
  const float scale = kLog2e * rsqrtf((float)kDh);
  if (mbar_wait(&mma1_bar, 0, &abort_s)) {
    tc_fence_after();
    const int slot = warp * 32 + lane;
    for (int h0 = 0; h0 < hp; h0 += 32) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)h0, r);
      tmem_ld_wait();
      const int nh = min(32, hp - h0);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j < nh) sS[(h0 + j) * kChunk + slot] = slot < n_valid ? __uint_as_float(r[j]) * scale : -INFINITY;
    }
    // slots that hold no position yet may hold anything (NaN included): their values are
    // zeroed so that the second product, where their weight is 0, stays finite
    if (n_valid < kChunk) {
      const int d = warp * 32 + lane;  // one row of Vᵀ per thread
      for (int k = n_valid; k < kChunk; ++k)
        *reinterpret_cast<__nv_bfloat16*>(sV + (k >> 6) * kDh * 128 + sw128_offset(d, k & 63)) =
            __float2bfloat16_rn(0.0f);
    }
  } else {
    ok = false;
    abort_s = 1;
    if (lane == 0) atomicOr(a.status, kStatusTimeout);
  }
  tc_fence_before();
  __syncthreads();
  // softmax numerators per head: warp w takes heads w, w + 4, …; lane l slots l + 32·i
  for (int h = warp; h < hp; h += 4) {
    float s[4];
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      s[i] = sS[h * kChunk + lane + 32 * i];
      m = fmaxf(m, s[i]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float l = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int k = lane + 32 * i;                   // slot within the chunk
      const __nv_bfloat16 p = __float2bfloat16_rn(exp2f(s[i] - m));   // exp2(−inf) = 0
      l += __bfloat162float(p);
      *reinterpret_cast<__nv_bfloat16*>(sP + (k >> 6) * hp * 128 + sw128_offset(h, k & 63)) = p;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    if (lane == 0 && h < a.H) {
      a.m_part[part * a.H + h] = m;
      a.l_part[part * a.H + h] = l;
    }
  }
  fence_proxy_async_smem();  // P is read by the tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && ok && !abort_s) {
    // Oᵀ[dim][head] = Σ_slot Vᵀ[dim][slot] P[head][slot]
    for (int kb = 0; kb < 2; ++kb)
      for (int k = 0; k < 4; ++k)
        umma_f16(tmem + (uint32_t)hp, umma_desc_sw128(smem_u32(sV + kb * kDh * 128) + k * 32),
                 umma_desc_sw128(smem_u32(sP + kb * hp * 128) + k * 32), idesc, (kb | k) != 0 ? 1u : 0u);
    umma_commit(&mma2_bar);
  }
  if (ok && mbar_wait(&mma2_bar, 0, &abort_s)) {
    tc_fence_after();
    const int d = warp * 32 + lane;
    for (int h0 = 0; h0 < hp; h0 += 32) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(hp + h0), r);
      tmem_ld_wait();
      const int nh = min(32, a.H - h0);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j < nh) a.o_part[(part * a.H + h0 + j) * kDh + d] = __uint_as_float(r[j]);
    }
  } else if (lane == 0) {
    atomicOr(a.status, kStatusTimeout);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

// ---- merge the chunks of each sequence ------------------------------------------------------
__global__ void __launch_bounds__(kDh) attn_combine_kernel(AttnArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.x, d = threadIdx.x;
  for (int h = blockIdx.y; h < a.H; h += gridDim.y) {
    float mx = -INFINITY;
    for (int c = 0; c < a.n_chunks; ++c) mx = fmaxf(mx, a.m_part[((int64_t)b * a.n_chunks + c) * a.H + h]);
    float num = 0.0f, den = 0.0f;
    for (int c = 0; c < a.n_chunks; ++c) {
      const int64_t part = (int64_t)b * a.n_chunks + c;
      const float l = a.l_part[part * a.H + h];
      if (l == 0.0f) continue;  // a chunk with no position of the window
      const float w = exp2f(a.m_part[part * a.H + h] - mx);
      num += w * a.o_part[(part * a.H + h) * kDh + d];
      den += w * l;
    }
    a.o[((int64_t)b * a.H + h) * kDh + d] = __float2bfloat16_rn(num / den);
  }
}

bool make_map_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1_bytes,
                 uint64_t s2_bytes, uint32_t b0, uint32_t b1) {
  EncodeTiledFn fn = get_encode_tiled();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1_bytes, s2_bytes};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename Kern, typename... Args>
cudaError_t launch_pdl(Kern k, dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, args...);
}

}  // namespace

AttnLayout attn_layout(int B, int D, int W) {
  AttnLayout L;
  L.H = D / kDh;
  L.n_chunks = W / kChunk;
  auto r256 = [](size_t n) { return (n + 255) / 256 * 256; };
  L.off_qkv = 256;  // [status word | pad]
  L.off_q = L.off_qkv + r256((size_t)B * (L.H + 2) * kDh * 2);
  L.off_op = L.off_q + r256((size_t)B * L.H * kDh * 2);
  L.off_m = L.off_op + r256((size_t)B * L.n_chunks * L.H * kDh * 4);
  L.off_l = L.off_m + r256((size_t)B * L.n_chunks * L.H * 4);
  L.off_o = L.off_l + r256((size_t)B * L.n_chunks * L.H * 4);
  L.bytes = L.off_o + r256((size_t)B * L.H * kDh * 2);
  return L;
}

cudaError_t launch_attention_core(const void* qkv, void* k_ring, void* v_ring, int64_t pos, int B, int D, int W,
                                  const AttnLayout& L, void* ws, unsigned* status, cudaStream_t s) {
  AttnArgs a{};
  uint8_t* w = static_cast<uint8_t*>(ws);
  a.qkv = static_cast<const __nv_bfloat16*>(qkv);
  a.q_rot = reinterpret_cast<__nv_bfloat16*>(w + L.off_q);
  a.k_ring = static_cast<__nv_bfloat16*>(k_ring);
  a.v_ring = static_cast<__nv_bfloat16*>(v_ring);
  a.o_part = reinterpret_cast<float*>(w + L.off_op);
  a.m_part = reinterpret_cast<float*>(w + L.off_m);
  a.l_part = reinterpret_cast<float*>(w + L.off_l);
  a.o = reinterpret_cast<__nv_bfloat16*>(w + L.off_o);
  a.status = status;
  a.pos = pos;
  a.B = B;
  a.H = L.H;
  a.W = W;
  a.n_chunks = L.n_chunks;
  CUtensorMap mk, mv, mq;
  if (!make_map_3d(&mk, k_ring, kDh, W, B, kDh * 2, (uint64_t)W * kDh * 2, 64, kChunk)) return cudaErrorInvalidValue;
  if (!make_map_3d(&mv, v_ring, W, kDh, B, (uint64_t)W * 2, (uint64_t)W * kDh * 2, 64, kDh))
    return cudaErrorInvalidValue;
  const AttnSmem sm = attn_smem(L.H);
  if (!make_map_3d(&mq, a.q_rot, kDh, L.H, B, kDh * 2, (uint64_t)L.H * kDh * 2, 64, (uint32_t)sm.hp))
    return cudaErrorInvalidValue;
  cudaError_t e = launch_pdl(attn_prep_kernel, dim3(B), dim3(256), 0, s, a);
  if (e != cudaSuccess) return e;
  static bool attr_set[64] = {};
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const size_t smem = (size_t)sm.bytes + 1024;
  if (!attr_set[dev]) {
    // the largest layout any call may need (kAttnMaxHeads query heads)
    e = cudaFuncSetAttribute(attn_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             attn_smem(kAttnMaxHeads).bytes + 1024);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  e = launch_pdl(attn_chunk_kernel, dim3(L.n_chunks, B), dim3(kAttnThreads), smem, s, mk, mv, mq, a);
  if (e != cudaSuccess) return e;
  const int hy = L.H < 8 ? L.H : 8;
  return launch_pdl(attn_combine_kernel, dim3(B, hy), dim3(kDh), 0, s, a);
}

}  // namespace rglru
