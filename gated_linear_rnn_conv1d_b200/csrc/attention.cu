// Decode step of Griffin's local multi-query attention on the sm_100a tensor cores.
//
// "Griffin：将门控线性循环与局部注意力混合以实现高效的语言模型", §时间混合块 (全局多查询注意力,
// 局部滑动窗口注意力): MQA (H query heads of D_head = 128, H·D_head = D, one key/value head
// shared by all of them), RoPE as the relative position embedding, local sliding-window
// attention (each position sees a fixed number of past positions, which bounds the KV cache
// by the window); "Griffin's Compromise: Combining Gated Linear Recurrence with Local
// Attention", §"Griffin: Attention for Recent Memory, Recurrence for Long-Range Flow":
// window 1024.
//
// One step at position `pos` for B sequences:
//   attn_prep_kernel   from the fused projection qkv = x W_qkvᵀ (or its split-K partial sums,
//                      which it adds up itself): rotates q and k (RoPE,
//                      pair i = (x_{2i}, x_{2i+1}) turned by pos·θ_i, θ_i = 10000^(−2i/128),
//                      the angle reduced in float64), writes the rotated queries, the key
//                      into slot (pos mod W) of the key ring and the value into the same
//                      slot of the (transposed) value ring;
//   attn_chunk_kernel  one CTA per (sequence, 128-slot chunk of the ring): TMA brings the
//                      chunk's keys and values [128 slots][128] and the sequence's queries
//                      [H][128] into 128-byte-swizzled shared memory;
//                      tcgen05.mma forms Sᵀ = K·Qᵀ (M = 128 slots, N = H heads, fp32 in
//                      TMEM); the four warps turn it into this chunk's softmax numerators
//                      P = 2^(s − m) (bf16, written in the swizzled layout the tensor core
//                      reads) with the chunk's per-head maximum m and sum l; a second MMA
//                      forms Oᵀ = Vᵀ·Pᵀ (M = 128 dims, N = H, Vᵀ read MN-major); the partial output, m and l
//                      go to the workspace. Slots not yet written (pos < W − 1) are masked.
//   attn_combine_kernel  merges the chunks of each sequence and head (flash-decoding):
//                      o = Σ_c 2^(m_c − m*) O_c / Σ_c 2^(m_c − m*) l_c, in bf16.
// The q, k, v and output projections run on the tcgen05 GEMM of gemm_tc.cu.
//
// Ring layouts: keys and values [B][W][128], slot-major (a chunk is one contiguous 32 KB
// block of each, and a step writes one 256-byte row of each). The attention is a sum over
// the window's slots, so they are read in slot order whatever position each holds. Every
// wait is bounded.
#include <cmath>
#include <cstdint>
#include <cuda_bf16.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace rglru {
namespace {

constexpr int kDh = 128;          // D_head
constexpr int kChunk = 128;       // ring slots per CTA
constexpr int kAttnThreads = 192;  // TMA warp, MMA warp, four softmax warps
constexpr float kLog2e = 1.4426950408889634f;

// Shared memory of the chunk kernel, offsets from a 1024-aligned base (every TMA box and
// operand tile starts 1024-aligned): two stages of [keys 2 × [128 slots][64 dims] | values
// 2 × [128 slots][64 dims] | queries 2 × [hp heads][64 dims]], then two buffers of softmax
// numerators P (2 k-blocks [hp][64 slots] each) and the scores [hp][128] float.
constexpr int kAttnStages = 2;
constexpr int kSPitch = kChunk + 4;  // floats per score row: 16-byte row reads stay conflict-free
struct AttnSmem {
  int hp;  // heads rounded up to 16 (the MMA's N)
  int stage, off_k, off_v, off_q, off_p, off_s, bytes;
};
__host__ __device__ inline AttnSmem attn_smem(int H) {
  AttnSmem L;
  L.hp = (H + 15) / 16 * 16;
  L.off_k = 0;
  L.off_v = L.off_k + 2 * kChunk * 128;
  L.off_q = L.off_v + 2 * kDh * 128;
  L.stage = L.off_q + ((2 * L.hp * 128 + 1023) / 1024) * 1024;
  L.off_p = kAttnStages * L.stage;  // two P buffers (items alternate)
  L.off_s = L.off_p + 2 * (((2 * L.hp * 128 + 1023) / 1024) * 1024);
  L.bytes = L.off_s + L.hp * kSPitch * 4;
  return L;
}

struct AttnArgs {
  const __nv_bfloat16* qkv;  // [B][(H+2)·128], or (when qkv_part is set) unused
  const float* qkv_part;     // [ksp][B][(H+2)·128]: the projection's split-K partial sums
  int ksp;
  int n_used;                // ring chunks holding a position of the window (all once it wrapped)
  __nv_bfloat16* q_rot;      // [B][H][128]
  __nv_bfloat16* k_ring;     // [B][W][128]
  __nv_bfloat16* v_ring;     // [B][W][128]
  float* o_part;             // [B][n_chunks][H][128]
  float* m_part;             // [B][n_chunks][H]
  float* l_part;             // [B][n_chunks][H]
  __nv_bfloat16* o;          // [B][H·128]
  unsigned* status;
  int64_t pos;
  int B, H, W, n_chunks;
};

// ---- RoPE, ring writes ------------------------------------------------------------------
// Grid (B, ⌈(H + 2)·32 / 512⌉): each thread takes two units of four consecutive columns of
// one sequence's projection row (a unit is two rotation pairs of one head), so that one
// wave of CTAs covers the batch. A column's value is qkv's bf16, or the bf16 rounding of
// the sum of the split-K slices (summed in slice order from 0, as the split GEMM's own
// reduction does), so both paths see the same bits. Every load a thread needs (up to four
// slices of both units at a time) is issued before the first add.
constexpr int kPrepThreads = 256;
constexpr int kPrepUnits = 2;   // four-column units per thread
constexpr int kPrepSlices = 4;  // slices requested together

__global__ void __launch_bounds__(kPrepThreads) attn_prep_kernel(AttnArgs a) {
  // the 64 rotation angles of this position (the same for every head and every sequence):
  // θ_j = 10000^(−2j/128), the angle pos·θ_j reduced modulo 2π in float64 so that large
  // positions keep their accuracy. They depend on nothing the projection writes, so they
  // are formed while it finishes.
  __shared__ float s_cos[kDh / 2], s_sin[kDh / 2];
  if (threadIdx.x < kDh / 2) {
    const int j = threadIdx.x;
    const double theta = exp(-(double)j * (2.0 / kDh) * 9.210340371976184);  // ln 10000
    const double ang = fmod((double)a.pos * theta, 6.283185307179586);
    double sd, cd;
    sincos(ang, &sd, &cd);
    s_cos[j] = (float)cd;
    s_sin[j] = (float)sd;
  }
  __syncthreads();
  pdl_wait();  // the projection is the previous kernel's output
  pdl_launch_dependents();
  const int b = blockIdx.x;
  const int H = a.H;
  const int64_t nq = (int64_t)(H + 2) * kDh;
  const int n_units = (H + 2) * (kDh / 4);
  const int unit0 = blockIdx.y * (kPrepThreads * kPrepUnits) + threadIdx.x;
  if (unit0 >= n_units) return;
  bool ok[kPrepUnits];
#pragma unroll
  for (int q = 0; q < kPrepUnits; ++q) ok[q] = unit0 + q * kPrepThreads < n_units;
  float x[kPrepUnits][4];
  if (a.qkv_part == nullptr) {
#pragma unroll
    for (int q = 0; q < kPrepUnits; ++q)
      if (ok[q]) {
        const uint2 v = *reinterpret_cast<const uint2*>(a.qkv + (int64_t)b * nq + (unit0 + q * kPrepThreads) * 4);
        x[q][0] = bf16lo(v.x); x[q][1] = bf16hi(v.x); x[q][2] = bf16lo(v.y); x[q][3] = bf16hi(v.y);
      }
  } else {
    const int64_t stride = (int64_t)a.B * nq;
    const float* src = a.qkv_part + (int64_t)b * nq + unit0 * 4;
    float4 acc[kPrepUnits];
#pragma unroll
    for (int q = 0; q < kPrepUnits; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < a.ksp; s0 += kPrepSlices) {
      float4 p[kPrepUnits][kPrepSlices];
#pragma unroll
      for (int q = 0; q < kPrepUnits; ++q)
#pragma unroll
        for (int j = 0; j < kPrepSlices; ++j)
          if (ok[q] && s0 + j < a.ksp)
            p[q][j] = __ldcs(reinterpret_cast<const float4*>(src + (s0 + j) * stride + q * kPrepThreads * 4));
#pragma unroll
      for (int q = 0; q < kPrepUnits; ++q)
#pragma unroll
        for (int j = 0; j < kPrepSlices; ++j)
          if (ok[q] && s0 + j < a.ksp) {
            acc[q].x += p[q][j].x;
            acc[q].y += p[q][j].y;
            acc[q].z += p[q][j].z;
            acc[q].w += p[q][j].w;
          }
    }
#pragma unroll
    for (int q = 0; q < kPrepUnits; ++q) {
      const uint32_t lo = pack_bf16x2(acc[q].x, acc[q].y), hi = pack_bf16x2(acc[q].z, acc[q].w);
      x[q][0] = bf16lo(lo); x[q][1] = bf16hi(lo); x[q][2] = bf16lo(hi); x[q][3] = bf16hi(hi);
    }
  }
  const int slot = (int)(a.pos % a.W);
#pragma unroll
  for (int q = 0; q < kPrepUnits; ++q) {
    if (!ok[q]) continue;
    const int col = (unit0 + q * kPrepThreads) * 4, head = col / kDh, j0 = (col % kDh) / 2;
    if (head == H + 1) {  // the value, unrotated, into the slot of the value ring
      *reinterpret_cast<uint2*>(a.v_ring + ((int64_t)b * a.W + slot) * kDh + col % kDh) =
          make_uint2(pack_bf16x2(x[q][0], x[q][1]), pack_bf16x2(x[q][2], x[q][3]));
      continue;
    }
    uint32_t r[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float sn = s_sin[j0 + e], cs = s_cos[j0 + e];
      const float x0 = x[q][2 * e], x1 = x[q][2 * e + 1];
      r[e] = pack_bf16x2(x0 * cs - x1 * sn, x0 * sn + x1 * cs);
    }
    __nv_bfloat16* dst = head < H ? a.q_rot + ((int64_t)b * H + head) * kDh
                                  : a.k_ring + ((int64_t)b * a.W + slot) * kDh;  // the key
    *reinterpret_cast<uint2*>(dst + col % kDh) = make_uint2(r[0], r[1]);
  }
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
__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ uint32_t sw128_offset(int row, int k) {
  return (uint32_t)row * 128u + ((uint32_t)((k >> 3) ^ (row & 7)) << 4) + (uint32_t)(k & 7) * 2u;
}

// Persistent: one CTA per SM walks the (sequence, chunk) items blockIdx.x, + gridDim.x, …
// Warp roles: 0 issues the TMA loads of item n into stage n mod 2 (two items ahead of the
// MMAs, so the next chunk streams in while this one is computed); 1 owns TMEM and issues the
// two MMAs of each item; 2–5 turn the scores into softmax numerators and write the partial
// outputs. The softmax warps run one item ahead of their outputs: item n's numerators are
// handed to the second MMA before item n − 1's output is read, so both MMAs' latency hides
// behind that work. Sᵀ and the score buffer are single; P and Oᵀ alternate between two
// buffers. Barriers: full/empty per stage; per item s_full (Sᵀ in TMEM) and p_full (P in
// shared memory); o_full per Oᵀ buffer. The orders that make the reuse safe:
//   Sᵀ(n) is written after p_full(n − 1), by which time the scores of n − 1 are read;
//   Oᵀ(n mod 2) is written after p_full(n), which the softmax warps give only after they
//   read Oᵀ(n − 2); P(n mod 2) is written after the softmax warps saw o_full(n − 2).
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_chunk_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmQ, AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kAttnStages], empty_bar[kAttnStages], o_full[2];
  __shared__ __align__(8) uint64_t s_full, p_full, drain_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const AttnSmem L = attn_smem(a.H);
  const int hp = L.hp;
  const int p_bytes = ((2 * hp * 128 + 1023) / 1024) * 1024;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_items = a.B * a.n_used;
  // Sᵀ in columns [0, hp), the two Oᵀ buffers in [hp, 3hp); 32 more so that every 32-column
  // load of the last group stays inside the allocation
  const int need = 3 * hp + 32;
  const uint32_t tmem_cols = need <= 64 ? 64u : (need <= 128 ? 128u : (need <= 256 ? 256u : 512u));
  static_assert(kAttnMaxHeads <= 64, "two stages, two P buffers and the scores fit in shared memory");

  if (threadIdx.x == 0) {
    for (int i = 0; i < kAttnStages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
      mbar_init(&o_full[i], 1);
    }
    mbar_init(&s_full, 1);
    mbar_init(&p_full, 4);  // one arrival per softmax warp
    mbar_init(&drain_bar, 1);
    abort_s = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_s, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();  // the rings and the rotated queries are the previous kernel's output
  pdl_launch_dependents();
  const uint32_t tmem = tmem_base_s;
  const uint32_t idesc = umma_idesc_bf16_f32(128, hp);

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmQ);
      const uint32_t bytes = 2 * kChunk * 128 + 2 * kDh * 128 + 2 * hp * 128;
      int n = 0;
      for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++n) {
        const int st = n % kAttnStages;
        if (n >= kAttnStages && !mbar_wait(&empty_bar[st], (uint32_t)((n / kAttnStages) - 1) & 1u, &abort_s)) {
          abort_s = 1;
          atomicOr(a.status, kStatusTimeout);
          break;
        }
        const int b = item / a.n_used, c = item % a.n_used;
        uint8_t* stage = smem + st * L.stage;
        mbar_arrive_expect_tx(&full_bar[st], bytes);
        for (int kb = 0; kb < 2; ++kb) {
          tma_load_3d(stage + L.off_k + kb * kChunk * 128, &tmK, &full_bar[st], kb * 64, c * kChunk, b);
          tma_load_3d(stage + L.off_v + kb * kChunk * 128, &tmV, &full_bar[st], kb * 64, c * kChunk, b);
          tma_load_3d(stage + L.off_q + kb * hp * 128, &tmQ, &full_bar[st], kb * 64, 0, b);  // rows ≥ H: 0
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int n = 0;
      for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++n) {
        const int st = n % kAttnStages;
        const uint8_t* stage = smem + st * L.stage;
        if (!mbar_wait(&full_bar[st], (uint32_t)(n / kAttnStages) & 1u, &abort_s)) break;
        tc_fence_after();
        // Sᵀ[slot][head] = Σ_d K[slot][d] Q[head][d]
        for (int kb = 0; kb < 2; ++kb)
          for (int k = 0; k < 4; ++k)
            umma_f16(tmem, umma_desc_sw128(smem_u32(stage + L.off_k + kb * kChunk * 128) + k * 32),
                     umma_desc_sw128(smem_u32(stage + L.off_q + kb * hp * 128) + k * 32), idesc,
                     (kb | k) != 0 ? 1u : 0u);
        umma_commit(&s_full);
        if (!mbar_wait(&p_full, (uint32_t)n & 1u, &abort_s)) break;
        tc_fence_after();
        // Oᵀ[dim][head] = Σ_slot Vᵀ[dim][slot] P[head][slot], into buffer n mod 2. The values
        // sit slot-major as loaded (rows of 64 dims per slot, the second 64 dims a box
        // further): Vᵀ is read as an MN-major operand, 16 slot rows per MMA.
        const uint8_t* pbuf = smem + L.off_p + (n & 1) * p_bytes;
        for (int kb = 0; kb < 2; ++kb)
          for (int k = 0; k < 4; ++k)
            umma_f16(tmem + (uint32_t)((1 + (n & 1)) * hp),
                     umma_desc_sw128_mn(smem_u32(stage + L.off_v) + (kb * 4 + k) * 2048, kChunk * 128),
                     umma_desc_sw128(smem_u32(pbuf + kb * hp * 128) + k * 32), idesc | kIdescAMN,
                     (kb | k) != 0 ? 1u : 0u);
        umma_commit(&o_full[n & 1]);
        umma_commit(&empty_bar[st]);  // the stage's operands are read
      }
      umma_commit(&drain_bar);
      volatile int never = 0;
      (void)mbar_wait(&drain_bar, 0, &never);
    }
  } else {
    // ---------------- softmax and outputs (warps 2–5) ----------------
    const int w4 = warp - 2;  // heads w4, w4 + 4, … of the softmax
    const int q4 = warp & 3;  // the TMEM lane quarter this warp may access: 32·(warp mod 4)
    float* sS = reinterpret_cast<float*>(smem + L.off_s);
    const float scale = kLog2e * rsqrtf((float)kDh);
    // the outputs of item `it` (the n-th of this CTA) from Oᵀ buffer n mod 2
    auto write_outputs = [&](int it, int n) -> bool {
      if (!mbar_wait(&o_full[n & 1], (uint32_t)(n >> 1) & 1u, &abort_s)) return false;
      tc_fence_after();
      const int64_t part = (int64_t)(it / a.n_used) * a.n_chunks + it % a.n_used;
      const int d = q4 * 32 + lane;
      for (int h0 = 0; h0 < hp; h0 += 32) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)((1 + (n & 1)) * hp + h0), r);
        tmem_ld_wait();
        const int nh = min(32, a.H - h0);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < nh) a.o_part[(part * a.H + h0 + j) * kDh + d] = __uint_as_float(r[j]);
      }
      tc_fence_before();
      return true;
    };
    int n = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++n) {
      const int st = n % kAttnStages;
      uint8_t* sV = smem + st * L.stage + L.off_v;
      uint8_t* sP = smem + L.off_p + (n & 1) * p_bytes;
      const int b = item / a.n_used, c = item % a.n_used;
      const int64_t part = (int64_t)b * a.n_chunks + c;
      const int64_t first = (int64_t)c * kChunk;
      const int n_valid =
          a.pos >= a.W - 1 ? kChunk : (int)max((int64_t)0, min((int64_t)kChunk, a.pos + 1 - first));
      if (!mbar_wait(&s_full, (uint32_t)n & 1u, &abort_s)) {
        if (lane == 0) atomicOr(a.status, kStatusTimeout);
        break;
      }
      tc_fence_after();
      if (n > 0) named_bar_sync(1, 128);  // every warp is done reading the previous scores
      // scores → sS[head][slot] in log2 units; slots holding no position: −inf
      const int slot = q4 * 32 + lane;
      for (int h0 = 0; h0 < hp; h0 += 32) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)h0, r);
        tmem_ld_wait();
        const int nh = min(32, hp - h0);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < nh) sS[(h0 + j) * kSPitch + slot] = slot < n_valid ? __uint_as_float(r[j]) * scale : -INFINITY;
      }
      // values of slots holding no position may be anything (NaN included): zeroed, so that
      // the second product, where their weight is 0, stays finite
      if (n_valid < kChunk) {
        const int d = q4 * 32 + lane;  // one value dimension per thread
        for (int k = n_valid; k < kChunk; ++k)
          *reinterpret_cast<__nv_bfloat16*>(sV + (d >> 6) * kChunk * 128 + sw128_offset(k, d & 63)) =
              __float2bfloat16_rn(0.0f);
      }
      tc_fence_before();
      named_bar_sync(1, 128);  // the scores of all 128 slots are in sS
      // softmax numerators: tph threads per head (8, 4 or 2), each over a run of
      // spt = 128 / tph slots, read as 16-byte rows and written as 16-byte chunks of P. A warp
      // holds hpw = 32 / tph heads; lane l takes head l mod hpw and run l / hpw, so that the
      // eight lanes of each 16-byte access phase touch eight rows (no bank conflicts) and a
      // head's runs meet in shuffles across lanes hpw, 2·hpw, … apart.
      {
        const int tph = hp <= 16 ? 8 : (hp <= 32 ? 4 : 2);
        const int spt = kChunk / tph;
        const int hpw = 32 / tph;
        const int h = w4 * hpw + lane % hpw, g = lane / hpw;
        if (w4 * hpw < hp) {  // whole warps drop out (hp is a multiple of 16 ≥ hpw)
          const float* row = sS + h * kSPitch + g * spt;
          float m = -INFINITY;
          for (int k = 0; k < spt; k += 4) {
            const float4 v = *reinterpret_cast<const float4*>(row + k);
            m = fmaxf(m, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
          }
          for (int off = hpw; off < 32; off <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
          float l = 0.0f;
          for (int k = 0; k < spt; k += 8) {
            const float4 v0 = *reinterpret_cast<const float4*>(row + k);
            const float4 v1 = *reinterpret_cast<const float4*>(row + k + 4);
            const float e[8] = {exp2f(v0.x - m), exp2f(v0.y - m), exp2f(v0.z - m), exp2f(v0.w - m),
                                exp2f(v1.x - m), exp2f(v1.y - m), exp2f(v1.z - m), exp2f(v1.w - m)};  // 2^−inf = 0
            uint32_t pk[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              pk[q] = pack_bf16x2(e[2 * q], e[2 * q + 1]);
              l += bf16lo(pk[q]) + bf16hi(pk[q]);  // the sum of the rounded numerators
            }
            const int kk = g * spt + k;  // the chunk's first slot
            *reinterpret_cast<uint4*>(sP + (kk >> 6) * hp * 128 + h * 128 + ((((kk & 63) >> 3) ^ (h & 7)) << 4)) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
          for (int off = hpw; off < 32; off <<= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
          if (g == 0 && h < a.H) {
            a.m_part[part * a.H + h] = m;
            a.l_part[part * a.H + h] = l;
          }
        }
      }
      fence_proxy_async_smem();  // P and the zeroed values are read by the tensor core
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full);
      // the previous item's outputs, while this item's second MMA runs
      if (n > 0 && !write_outputs(item - (int)gridDim.x, n - 1)) {
        if (lane == 0) atomicOr(a.status, kStatusTimeout);
        ok = false;
      }
    }
    if (ok && n > 0 && !write_outputs(blockIdx.x + (n - 1) * (int)gridDim.x, n - 1)) {
      if (lane == 0) atomicOr(a.status, kStatusTimeout);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

// ---- merge the chunks of each sequence ------------------------------------------------------
// One warp per (sequence, head), four output dimensions per lane (16-byte loads of the partial
// outputs), eight heads per CTA. The chunks' maxima are spread over the lanes and reduced by
// shuffles; then every lane walks the chunks in order with their weights 2^(m_c − m*) (the
// same arithmetic, in the same order, for every dimension). Chunks are fetched eight at a
// time, the first eight together with the maxima, so that a window of up to 1024 slots costs
// one round trip to memory.
constexpr int kCombineHeads = 8;
constexpr int kCombineBatch = 8;
__global__ void __launch_bounds__(32 * kCombineHeads) attn_combine_kernel(AttnArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.x, h = blockIdx.y * kCombineHeads + (int)threadIdx.x / 32, lane = threadIdx.x % 32;
  if (h >= a.H) return;
  const int64_t base = (int64_t)b * a.n_chunks;
  const int n = a.n_used;
  float4 o[kCombineBatch];
  float mc[kCombineBatch], lc[kCombineBatch];
  auto fetch = [&](int c0) {
#pragma unroll
    for (int j = 0; j < kCombineBatch; ++j)
      if (c0 + j < n) {
        const int64_t part = base + c0 + j;
        mc[j] = a.m_part[part * a.H + h];
        lc[j] = a.l_part[part * a.H + h];
        o[j] = *reinterpret_cast<const float4*>(a.o_part + (part * a.H + h) * kDh + 4 * lane);
      }
  };
  fetch(0);
  float mx = -INFINITY;
  for (int c = lane; c < n; c += 32) mx = fmaxf(mx, a.m_part[(base + c) * a.H + h]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.0f;
  for (int c0 = 0;;) {
#pragma unroll
    for (int j = 0; j < kCombineBatch; ++j)
      if (c0 + j < n) {
        const float w = exp2f(mc[j] - mx);
        num = make_float4(fmaf(w, o[j].x, num.x), fmaf(w, o[j].y, num.y), fmaf(w, o[j].z, num.z),
                          fmaf(w, o[j].w, num.w));
        den = fmaf(w, lc[j], den);
      }
    c0 += kCombineBatch;
    if (c0 >= n) break;
    fetch(c0);
  }
  *reinterpret_cast<uint2*>(a.o + ((int64_t)b * a.H + h) * kDh + 4 * lane) =
      make_uint2(pack_bf16x2(num.x / den, num.y / den), pack_bf16x2(num.z / den, num.w / den));
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
  L.off_part = L.off_o + r256((size_t)B * L.H * kDh * 2);
  L.bytes = L.off_part + kSplitPartBytes;
  return L;
}

cudaError_t launch_attention_core(const void* qkv, const float* qkv_part, int ksp, void* k_ring, void* v_ring,
                                  int64_t pos, int B, int D, int W, const AttnLayout& L, void* ws, unsigned* status,
                                  cudaStream_t s) {
  AttnArgs a{};
  uint8_t* w = static_cast<uint8_t*>(ws);
  a.qkv = static_cast<const __nv_bfloat16*>(qkv);
  a.qkv_part = qkv_part;
  a.ksp = ksp;
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
  a.n_used = pos >= W - 1 ? L.n_chunks : (int)((pos + kChunk) / kChunk);  // chunks with a position
  CUtensorMap mk, mv, mq;
  if (!make_map_3d(&mk, k_ring, kDh, W, B, kDh * 2, (uint64_t)W * kDh * 2, 64, kChunk)) return cudaErrorInvalidValue;
  if (!make_map_3d(&mv, v_ring, kDh, W, B, kDh * 2, (uint64_t)W * kDh * 2, 64, kChunk))
    return cudaErrorInvalidValue;
  const AttnSmem sm = attn_smem(L.H);
  if (!make_map_3d(&mq, a.q_rot, kDh, L.H, B, kDh * 2, (uint64_t)L.H * kDh * 2, 64, (uint32_t)sm.hp))
    return cudaErrorInvalidValue;
  const int prep_blocks = ((L.H + 2) * (kDh / 4) + kPrepThreads * kPrepUnits - 1) / (kPrepThreads * kPrepUnits);
  cudaError_t e = launch_pdl(attn_prep_kernel, dim3(B, prep_blocks), dim3(kPrepThreads), 0, s, a);
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
  const int items = B * a.n_used;
  const int grid = items < num_sms() ? items : num_sms();
  e = launch_pdl(attn_chunk_kernel, dim3(grid), dim3(kAttnThreads), smem, s, mk, mv, mq, a);
  if (e != cudaSuccess) return e;
  return launch_pdl(attn_combine_kernel, dim3(B, (L.H + kCombineHeads - 1) / kCombineHeads),
                    dim3(32 * kCombineHeads), 0, s, a);
}

}  // namespace rglru
