// bf16 GEMMs on the sm_100a tensor cores (tcgen05.mma, fp32 accumulators in TMEM,
// operands staged by TMA into 128-byte-swizzled shared memory; no cluster multicast).
//
// Uses: the RG-LRU gate projections z = u [W_a | W_x]ᵀ + b ("Griffin：将门控线性循环与
// 局部注意力混合以实现高效的语言模型", §实门线性循环单元 (RG-LRU), Eq. (1)–(2)) — the only dense
// contraction of the layer — for prefill (packed z out) and for decode (the RG-LRU update
// fused into the epilogue, Eq. (3)–(4)); and the recurrent block's D ↔ D_RNN linears
// (§循环块).
//
// Kernel shape: persistent CTAs (one per SM), 192 threads.
//   warp 0      one lane issues TMA loads of A [128×64] and B [BN×64] k-blocks into a
//               ring of smem stages (full/empty mbarriers);
//   warp 1      allocates TMEM (two BN-column accumulators) and one lane issues
//               tcgen05.mma M=128, N=BN, K=16 (four per k-block), committing each stage
//               back to the producer and each finished tile to the epilogue;
//   warps 2–5   epilogue: tcgen05.ld of their 32 TMEM lanes (= 32 output rows), fused
//               element-wise work, global stores; the accumulator is handed back so the
//               next tile's MMAs overlap this tile's epilogue.
// "Dual" B: the gate GEMMs fetch the first BN/2 rows of a B tile from W_a and the second
// BN/2 from W_x (two tensor maps), so one tile holds both gates of the same channels.
#include <algorithm>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <mutex>

#include "gate_math.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace rglru {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;  // 64 bf16 = one 128-byte swizzle row
constexpr int kGemmThreads = 192;

enum EpiKind { EPI_STORE = 0, EPI_GATES = 1, EPI_STEP = 2, EPI_SCAN = 3, EPI_COEF = 4, EPI_STORE_F32 = 5 };

struct EpiArgs {
  __nv_bfloat16* C;   // STORE / GATES output
  float* Cf;          // STORE_F32 output
  int64_t ldc;        // elements
  int N;              // STORE: valid columns
  const float* b_a;   // GATES / STEP
  const float* b_x;
  int R;              // channels (GATES / STEP)
  const float* u;          // STEP: u_t [M][R] float32 (the GEMM read its bf16 rounding)
  float* h;                // STEP: state [M][R], in place
  __nv_bfloat16* y;        // STEP: y_t [M][R]
  const float* cla;        // STEP: c·log σ(Λ) [R]
  const __nv_bfloat16* ub; // COEF: u [M][R] bf16, the GEMM's A operand (b_t = m·u_t)
  // SCAN (gate GEMM fused with the RG-LRU scan):
  const __nv_bfloat16* x;       // [B][T][R] Conv1D input (u is recomputed from it in float32)
  const __nv_bfloat16* state0;  // [B][3][R] conv history or null
  const float* conv_w;          // [4][R]
  const float* conv_b;          // [R]
  const float* Lambda;          // [R]
  const float* h0;              // [B][R] or null
  float* hT;                    // [B][R] or null
  uint64_t* carry_agg;          // [B·n_nb·n_chunks][128] aggregates (zero at launch)
  uint32_t* carry_incl;         // [B·n_nb·n_chunks][128] inclusive states (zero at launch)
  int T, n_chunks;              // n_chunks = T / 128
  // STORE_F32 split over K: tile index = output tile · k_split + slice; slice s covers k-blocks
  // [s·kb_per, (s+1)·kb_per) and writes its partial sums at Cf + s·split_stride
  int k_split, kb_per;
  int64_t split_stride;
  // operands MN-major (STORE_F32, one B): A [K][M] (a_mn) and B [K][N] (b_mn) row-major,
  // staged as K rows of 64 M (N) columns; otherwise K-major, A [M][K] and B [N][K]. With
  // b_split_k > 0 (a multiple of BK), B's rows k ≥ b_split_k come from the second B map, at
  // row k − b_split_k: B = [B0; B1] stacked along K.
  int a_mn, b_mn, b_split_k;
  // COEF: the pre-activations z (with biases, bf16, the packed layout of C) stored as well
  // when not null — bit for bit what EPI_GATES writes for the same operands
  __nv_bfloat16* z_out;
  // STORE_F32: C += A·Bᵀ (C read before it is written, element by element) instead of C = A·Bᵀ
  int accumulate;
};

// The k-block range of slice `ks` (the whole K when the GEMM is not split).
__device__ __forceinline__ void kb_range(const EpiArgs& ep, int ks, int k_blocks, int& kb0, int& kb1) {
  if (ep.k_split > 1) {
    kb0 = ks * ep.kb_per;
    kb1 = min(k_blocks, kb0 + ep.kb_per);
  } else {
    kb0 = 0;
    kb1 = k_blocks;
  }
}

template <int BN> struct GemmCfg {
  static constexpr int kStages = BN == 256 ? 4 : 6;
  static constexpr int kABytes = BM * BK * 2;
  static constexpr int kBBytes = BN * BK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kSmem = kStages * kStageBytes + 1024;  // + alignment slack
  static constexpr int kTmemCols = 2 * BN;
  static constexpr uint32_t kIdesc = umma_idesc_bf16_f32(BM, BN);
};

__device__ __forceinline__ void store_row_bf16(__nv_bfloat16* dst, const float (&v)[32]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    d[q] = make_uint4(pack_bf16x2(v[8 * q + 0], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                      pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
}

template <int BN, int EPI, bool DUAL>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmB1, int64_t M, int K, int n_tiles_n, int num_tiles,
                   EpiArgs ep, unsigned* status) {
  using Cfg = GemmCfg<BN>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[S];
  __shared__ __align__(8) uint64_t empty_bar[S];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull_bar[i], 1);
      mbar_init(&tempty_bar[i], 4);
    }
    mbar_init(&drain_bar, 1);
    abort_s = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    if (DUAL) tma_prefetch_desc(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_s, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_s;
  const int k_blocks = (K + BK - 1) / BK;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m_blk = tile / n_tiles_n, n_blk = tile % n_tiles_n;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, &abort_s)) { ok = false; break; }
          uint8_t* sa = smem + stage * Cfg::kStageBytes;
          uint8_t* sb = sa + Cfg::kABytes;
          mbar_arrive_expect_tx(&full_bar[stage], Cfg::kStageBytes);
          tma_load_2d(sa, &tmA, &full_bar[stage], kb * BK, m_blk * BM);
          if (DUAL) {
            tma_load_2d(sb, &tmB0, &full_bar[stage], kb * BK, n_blk * (BN / 2));
            tma_load_2d(sb + (BN / 2) * BK * 2, &tmB1, &full_bar[stage], kb * BK, n_blk * (BN / 2));
          } else {
            tma_load_2d(sb, &tmB0, &full_bar[stage], kb * BK, n_blk * BN);
          }
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) { abort_s = 1; atomicOr(status, kStatusTimeout); }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1, &abort_s)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, &abort_s)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * Cfg::kStageBytes);
          const uint32_t b_addr = a_addr + Cfg::kABytes;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            umma_f16(d_tmem, umma_desc_sw128(a_addr + k * 32), umma_desc_sw128(b_addr + k * 32), Cfg::kIdesc,
                     (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit(&empty_bar[stage]);
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit(&tfull_bar[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      if (!ok) {
        abort_s = 1;
        atomicOr(status, kStatusTimeout);
      }
      // Drain: wait until every MMA issued by this thread has completed before TMEM is
      // freed (a barrier of its own, so the epilogue's phases are not disturbed).
      umma_commit(&drain_bar);
      {
        volatile int never = 0;
        (void)mbar_wait(&drain_bar, 0, &never);
      }
    }
  } else {
    // ---------------- epilogue warps ----------------
    const int quarter = warp & 3;  // a warp may only touch TMEM lanes 32*(warp%4) .. +31
    const int row_in_tile = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int m_blk = tile / n_tiles_n, n_blk = tile % n_tiles_n;
      if (!mbar_wait(&tfull_bar[acc], acc_phase, &abort_s)) {
        abort_s = 1;
        atomicOr(status, kStatusTimeout);
        break;
      }
      tc_fence_after();
      const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN;
      const int64_t row = (int64_t)m_blk * BM + row_in_tile;
      const bool row_ok = row < M;

      if constexpr (EPI == EPI_STORE || EPI == EPI_GATES) {
#pragma unroll 1
        for (int cc = 0; cc < BN / 32; ++cc) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(t_row + cc * 32, r);
          tmem_ld_wait();
          float v[32];
          const int col0 = cc * 32;
          if constexpr (EPI == EPI_GATES) {
            // packed layout: block n_blk holds channels [n_blk*BN/2, +BN/2), z_a then z_x
            const int half = col0 / (BN / 2);
            const int ch0 = n_blk * (BN / 2) + (col0 % (BN / 2));
            const float* bias = half ? ep.b_x : ep.b_a;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int ch = ch0 + j;
              v[j] = __uint_as_float(r[j]) + (ch < ep.R ? __ldg(bias + ch) : 0.0f);
            }
            if (row_ok) store_row_bf16(ep.C + row * ep.ldc + (int64_t)n_blk * BN + col0, v);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
            const int gcol = n_blk * BN + col0;
            if (row_ok) {
              if (gcol + 32 <= ep.N) {
                store_row_bf16(ep.C + row * ep.ldc + gcol, v);
              } else {
                uint4* d = reinterpret_cast<uint4*>(ep.C + row * ep.ldc + gcol);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  if (gcol + 8 * q < ep.N)
                    d[q] = make_uint4(pack_bf16x2(v[8 * q + 0], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                                      pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
              }
            }
          }
        }
      } else {
        // EPI_STEP: columns [0, BN/2) are z_a and [BN/2, BN) are z_x of channels
        // n_blk*BN/2 + j; row = batch index. h ← a_t h + √(1−a_t²) i u ; y = h.
#pragma unroll 1
        for (int cc = 0; cc < BN / 64; ++cc) {
          uint32_t ra[32], rx[32];
          tmem_ld_32x32b_x32(t_row + cc * 32, ra);
          tmem_ld_32x32b_x32(t_row + BN / 2 + cc * 32, rx);
          tmem_ld_wait();
          const int ch0 = n_blk * (BN / 2) + cc * 32;
          if (row_ok) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int c = ch0 + 8 * q;
              if (c < ep.R) {
                const float4* up = reinterpret_cast<const float4*>(ep.u + row * ep.R + c);
                const float4 u0 = up[0], u1 = up[1];
                float4* hp = reinterpret_cast<float4*>(ep.h + row * ep.R + c);
                const float4 h0 = hp[0], h1 = hp[1];
                float uu[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
                float hh[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                  const int ch = c + j;
                  const float za = __uint_as_float(ra[8 * q + j]) + __ldg(ep.b_a + ch);
                  const float zx = __uint_as_float(rx[8 * q + j]) + __ldg(ep.b_x + ch);
                  float at, bt;
                  gate_fast(za, zx, __ldg(ep.cla + ch), uu[j], at, bt);
                  hh[j] = fmaf(at, hh[j], bt);
                }
                hp[0] = make_float4(hh[0], hh[1], hh[2], hh[3]);
                hp[1] = make_float4(hh[4], hh[5], hh[6], hh[7]);
                *reinterpret_cast<uint4*>(ep.y + row * ep.R + c) =
                    make_uint4(pack_bf16x2(hh[0], hh[1]), pack_bf16x2(hh[2], hh[3]), pack_bf16x2(hh[4], hh[5]),
                               pack_bf16x2(hh[6], hh[7]));
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

// ---------------------------------------------------------------------------------------
// 2-SM form (cta_group::2): a cluster of two CTAs computes a 256×256 tile. Each CTA stages
// its own 128 rows of A and its own half of the B tile (128 rows); the leader CTA (rank 0)
// issues tcgen05.mma.cta_group::2 with M = 256, N = 256, which reads both CTAs' shared
// memory and leaves rows 0–127 of the tile in the leader's TMEM and rows 128–255 in the
// peer's. Per SM this halves the B bytes pulled from L2 per FLOP. Loads carry no
// multicast: both CTAs' TMA copies signal the leader's full barrier; the leader's commits
// are multicast (tcgen05.commit, not a load) to both CTAs' empty / accumulator barriers.
constexpr int k2Stages = 6;
constexpr int k2ABytes = BM * BK * 2;            // 16 KB: this CTA's 128 rows of A
constexpr int k2BBytes = 128 * BK * 2;           // 16 KB: this CTA's half of the B tile
constexpr int k2StageBytes = k2ABytes + k2BBytes;
constexpr int k2TmemCols = 512;                  // two 256-column accumulators
constexpr uint32_t k2Idesc = umma_idesc_bf16_f32(256, 256);

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t mapa_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void tma_load_2d_2sm(void* dst, const CUtensorMap* m, uint32_t leader_bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(leader_bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void umma_f16_2sm(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit_2sm_both(uint64_t* bar) {
  const uint16_t mask = 0x3;
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "h"(mask)
               : "memory");
}

// Fused-scan epilogue scratch after the pipeline stages: per tile parity the 128 channels'
// b_a, b_x and c·log σ(Λ); the four quarters' maps (A, B) per channel; their incoming states.
constexpr int kScanParBytes = 2 * 3 * 128 * 4;
constexpr int kScanTPitch = 17;  // float2 per row of a warp's transpose buffer (conflict-light)
constexpr int kScanTBytes = 8 * 32 * kScanTPitch * 8;  // eight warps × [32 rows][17] float2
constexpr int kScanEpiBytes = kScanParBytes + 4 * 128 * 8 + 4 * 128 * 4 + kScanTBytes;
constexpr int kScanStages = 5;  // (the transpose buffers take the sixth stage's room)
template <int EPI> __host__ __device__ constexpr int stages_of() { return EPI == EPI_SCAN ? kScanStages : k2Stages; }
constexpr int kCoefEpiBytes = 2 * 3 * 128 * 4;  // per tile parity: b_a, b_x, c·log σ(Λ) of 128 channels
// warps: 0 TMA, 1 MMA, then epilogue warps — 4 (one per TMEM lane quarter), or 8 for the
// coefficient epilogue (two per quarter, each taking half of the channels)
template <int EPI> __host__ __device__ constexpr int epi_warps_of() {
  return (EPI == EPI_COEF || EPI == EPI_SCAN) ? 8 : 4;
}
template <int EPI> __host__ __device__ constexpr int threads_of() { return 64 + 32 * epi_warps_of<EPI>(); }
template <int EPI> __host__ __device__ constexpr int smem_of() {
  return stages_of<EPI>() * k2StageBytes + (EPI == EPI_SCAN ? kScanEpiBytes : 0) +
         (EPI == EPI_COEF ? kCoefEpiBytes : 0) + 1024;
}

// Gate math for two elements: d = 1 − a_t and b_t = √(1−a_t²)·i·u, with r = σ(z_a),
// log a_t = r·cla, d = −expm1(log a_t) (Taylor polynomial to degree 6 on [−1/8, 0], 1 − ex2
// beyond), 1 − a_t² = d(2 − d), √(1−a_t²)·i = q·rsqrt(q (1 + e^{−z_x})² + 1e-30).
__device__ __forceinline__ void gate_fast2_pair(float2 za, float2 zx, float2 cla, float2 u, float2& d, float2& bt) {
  const float2 na = __fmul2_rn(za, make_float2(-kLog2e, -kLog2e));
  const float2 nx = __fmul2_rn(zx, make_float2(-kLog2e, -kLog2e));
  const float2 ea = __fadd2_rn(make_float2(ex2_approx(na.x), ex2_approx(na.y)), make_float2(1.0f, 1.0f));
  const float2 r = make_float2(rcp_approx(ea.x), rcp_approx(ea.y));
  const float2 la = __fmul2_rn(r, cla);
  if (fminf(la.x, la.y) >= -0.125f) {
    float2 p = __ffma2_rn(la, make_float2(1.0f / 720.0f, 1.0f / 720.0f), make_float2(1.0f / 120.0f, 1.0f / 120.0f));
    p = __ffma2_rn(p, la, make_float2(1.0f / 24.0f, 1.0f / 24.0f));
    p = __ffma2_rn(p, la, make_float2(1.0f / 6.0f, 1.0f / 6.0f));
    p = __ffma2_rn(p, la, make_float2(0.5f, 0.5f));
    p = __ffma2_rn(p, la, make_float2(1.0f, 1.0f));
    d = __fmul2_rn(make_float2(-la.x, -la.y), p);
  } else {
    d.x = la.x >= -0.125f ? neg_expm1_small(la.x) : 1.0f - ex2_approx(la.x * kLog2e);
    d.y = la.y >= -0.125f ? neg_expm1_small(la.y) : 1.0f - ex2_approx(la.y * kLog2e);
  }
  const float2 q = __fmul2_rn(d, __fadd2_rn(make_float2(2.0f, 2.0f), make_float2(-d.x, -d.y)));
  const float2 t1 = __fadd2_rn(make_float2(ex2_approx(nx.x), ex2_approx(nx.y)), make_float2(1.0f, 1.0f));
  const float2 dd = __ffma2_rn(__fmul2_rn(q, t1), t1, make_float2(1e-30f, 1e-30f));
  const float2 rs = make_float2(rsqrt_approx(dd.x), rsqrt_approx(dd.y));
  bt = __fmul2_rn(__fmul2_rn(q, rs), u);
}

__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ uint32_t ld_relaxed_u32g(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint64_t ld_relaxed_u64g(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u32g(uint32_t* p, uint32_t v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void st_relaxed_u64g(uint64_t* p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
// Published carries are stored as their bit pattern XOR 0x7FFFFFFF: exact and reversible,
// and zero only for one NaN pattern, so zeroed memory reads as "not published yet".
// (the NaN pattern 0x7FFFFFFF, whose image would be zero, is stored as another NaN's image)
__device__ __forceinline__ uint32_t enc_carry(float v) {
  const uint32_t w = __float_as_uint(v) ^ 0x7FFFFFFFu;
  return w != 0u ? w : 1u;
}
__device__ __forceinline__ float dec_carry(uint32_t w) { return __uint_as_float(w ^ 0x7FFFFFFFu); }


// 16 columns of this warp's TMEM lane quarter; the values are valid only after
// tmem_ld_wait16 on the same registers (which ties every use to the wait).
__device__ __forceinline__ void tmem_ld_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait16(uint32_t (&a)[16], uint32_t (&b)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(a[0]), "+r"(a[1]), "+r"(a[2]), "+r"(a[3]), "+r"(a[4]), "+r"(a[5]), "+r"(a[6]), "+r"(a[7]),
                 "+r"(a[8]), "+r"(a[9]), "+r"(a[10]), "+r"(a[11]), "+r"(a[12]), "+r"(a[13]), "+r"(a[14]),
                 "+r"(a[15]), "+r"(b[0]), "+r"(b[1]), "+r"(b[2]), "+r"(b[3]), "+r"(b[4]), "+r"(b[5]), "+r"(b[6]),
                 "+r"(b[7]), "+r"(b[8]), "+r"(b[9]), "+r"(b[10]), "+r"(b[11]), "+r"(b[12]), "+r"(b[13]),
                 "+r"(b[14]), "+r"(b[15])
               :
               : "memory");
}

template <int EPI, bool DUAL>
__global__ void __launch_bounds__(threads_of<EPI>(), 1)
    gemm2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                 const __grid_constant__ CUtensorMap tmB1, int64_t M, int K, int n_tiles_n, int num_tiles, EpiArgs ep,
                 unsigned* status) {
  constexpr int S = stages_of<EPI>();
  constexpr int BN = 256;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[S];
  __shared__ __align__(8) uint64_t empty_bar[S];
  __shared__ __align__(8) uint64_t tfull_bar[2];
  __shared__ __align__(8) uint64_t tempty_bar[2];
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = blockIdx.x / 2;
  const int n_clusters = gridDim.x / 2;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull_bar[i], 1);
      mbar_init(&tempty_bar[i], 2 * epi_warps_of<EPI>());  // the epilogue warps of both CTAs
    }
    mbar_init(&drain_bar, 1);
    abort_s = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    if (DUAL) tma_prefetch_desc(&tmB1);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_s)),
                 "r"(k2TmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  // launched as a programmatic dependent: everything above overlapped the previous kernel;
  // its results (the A operand, or anything else an epilogue reads) are visible from here
  pdl_wait();
  pdl_launch_dependents();
  const uint32_t tmem_base = tmem_base_s;
  const int k_blocks = (K + BK - 1) / BK;
  const uint32_t leader_full0 = mapa_rank(smem_u32(&full_bar[0]), 0);

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs) ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = cluster; tile < num_tiles && ok; tile += n_clusters) {
        const int ksp = ep.k_split > 1 ? ep.k_split : 1;
        const int tt = tile / ksp;
        const int m_pair = tt / n_tiles_n, n_blk = tt % n_tiles_n;
        const int arow = m_pair * 256 + (int)rank * 128;
        int kb0, kb1;
        kb_range(ep, tile % ksp, k_blocks, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, &abort_s)) { ok = false; break; }
          uint8_t* sa = smem + stage * k2StageBytes;
          uint8_t* sb = sa + k2ABytes;
          const uint32_t lbar = leader_full0 + stage * 8;
          if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2 * k2StageBytes);
          if (!DUAL && (ep.a_mn | ep.b_mn)) {
            // an MN-major operand: this CTA's 128 columns as two boxes of 64 columns × BK rows
            if (ep.a_mn) {
              tma_load_2d_2sm(sa, &tmA, lbar, arow, kb * BK);
              tma_load_2d_2sm(sa + k2ABytes / 2, &tmA, lbar, arow + 64, kb * BK);
            } else {
              tma_load_2d_2sm(sa, &tmA, lbar, kb * BK, arow);
            }
            const int bcol = n_blk * 256 + (int)rank * 128;
            if (ep.b_mn) {
              const bool second = ep.b_split_k > 0 && kb * BK >= ep.b_split_k;
              const CUtensorMap* mb = second ? &tmB1 : &tmB0;
              const int kr = kb * BK - (second ? ep.b_split_k : 0);
              tma_load_2d_2sm(sb, mb, lbar, bcol, kr);
              tma_load_2d_2sm(sb + k2BBytes / 2, mb, lbar, bcol + 64, kr);
            } else {
              tma_load_2d_2sm(sb, &tmB0, lbar, kb * BK, bcol);
            }
          } else if (DUAL) {
            tma_load_2d_2sm(sa, &tmA, lbar, kb * BK, arow);
            tma_load_2d_2sm(sb, rank == 0 ? &tmB0 : &tmB1, lbar, kb * BK, n_blk * 128);
          } else {
            tma_load_2d_2sm(sa, &tmA, lbar, kb * BK, arow);
            tma_load_2d_2sm(sb, &tmB0, lbar, kb * BK, n_blk * 256 + (int)rank * 128);
          }
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) { abort_s = 1; atomicOr(status, kStatusTimeout); }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader CTA only) ----------------
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = cluster; tile < num_tiles && ok; tile += n_clusters) {
        if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1, &abort_s)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        int kb0, kb1;
        kb_range(ep, tile % (ep.k_split > 1 ? ep.k_split : 1), k_blocks, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, &abort_s)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * k2StageBytes);
          const uint32_t b_addr = a_addr + k2ABytes;
          if (!DUAL && (ep.a_mn | ep.b_mn)) {
            // MN-major: 16 k-rows of 128 B per MMA, the second 64 columns half a stage operand
            // further; K-major: 32 bytes further along the swizzled rows
            const uint32_t idesc = k2Idesc | (ep.a_mn ? kIdescAMN : 0u) | (ep.b_mn ? kIdescBMN : 0u);
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              umma_f16_2sm(d_tmem,
                           ep.a_mn ? umma_desc_sw128_mn(a_addr + k * 2048, k2ABytes / 2)
                                   : umma_desc_sw128(a_addr + k * 32),
                           ep.b_mn ? umma_desc_sw128_mn(b_addr + k * 2048, k2BBytes / 2)
                                   : umma_desc_sw128(b_addr + k * 32),
                           idesc, (kb != kb0 || k != 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              umma_f16_2sm(d_tmem, umma_desc_sw128(a_addr + k * 32), umma_desc_sw128(b_addr + k * 32), k2Idesc,
                           (kb != kb0 || k != 0) ? 1u : 0u);
          }
          umma_commit_2sm_both(&empty_bar[stage]);
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit_2sm_both(&tfull_bar[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      if (!ok) { abort_s = 1; atomicOr(status, kStatusTimeout); }
      asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                       smem_u32(&drain_bar))
                   : "memory");
      volatile int never = 0;
      (void)mbar_wait(&drain_bar, 0, &never);
    }
  } else if constexpr (EPI != EPI_SCAN) {
    // ---------------- epilogue warps (both CTAs) ----------------
    const int quarter = warp & 3;
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t leader_tempty0 = mapa_rank(smem_u32(&tempty_bar[0]), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = cluster; tile < num_tiles; tile += n_clusters) {
      const int ksp = ep.k_split > 1 ? ep.k_split : 1;
      const int tt = tile / ksp;
      const int m_pair = tt / n_tiles_n, n_blk = tt % n_tiles_n;
      [[maybe_unused]] const int64_t split_off = (int64_t)(tile % ksp) * ep.split_stride;
      const int64_t row = (int64_t)m_pair * 256 + rank * 128 + row_in_tile;
      const bool row_ok = row < M;
      // COEF: this thread's 64 values of u_t (its row, its half of the tile's channels),
      // loaded before the accumulator is ready; 8 channels are all valid or all not (R % 8 = 0)
      [[maybe_unused]] uint4 uq[EPI == EPI_COEF ? 8 : 1];
      if constexpr (EPI == EPI_COEF) {
        const int ch0 = n_blk * 128 + ((warp - 2) / 4) * 64;
        const __nv_bfloat16* urow = ep.ub + row * ep.R + ch0;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          uq[q] = (row_ok && ch0 + 8 * q < ep.R) ? __ldg(reinterpret_cast<const uint4*>(urow) + q)
                                                 : make_uint4(0u, 0u, 0u, 0u);
        // the tile's channel parameters (b_a, b_x, c·log σ(Λ)), also before the accumulator
        // is ready: this parity's buffer was last read by the tile two back, which every
        // epilogue warp has finished (they all passed the previous tile's barrier)
        float* sPar = reinterpret_cast<float*>(smem + S * k2StageBytes) + acc * 3 * 128;
        if ((warp - 2) / 4 == 0) {
          const int ch = n_blk * 128 + row_in_tile;
          const bool ok = ch < ep.R;
          sPar[row_in_tile] = ok ? __ldg(ep.b_a + ch) : 0.0f;
          sPar[128 + row_in_tile] = ok ? __ldg(ep.b_x + ch) : 0.0f;
          sPar[256 + row_in_tile] = ok ? decay_log_coeff(__ldg(ep.Lambda + ch)) : 0.0f;
        }
      }
      if (!mbar_wait(&tfull_bar[acc], acc_phase, &abort_s)) {
        abort_s = 1;
        atomicOr(status, kStatusTimeout);
        break;
      }
      tc_fence_after();
      const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN;
      if constexpr (EPI == EPI_COEF) {
        // "Griffin：将门控线性循环与局部注意力混合以实现高效的语言模型", §实门线性循环单元, Eq. (3)–(4):
        // columns [0, 128) are z_a and [128, 256) z_x of channels n_blk·128 + j. Each row's
        // pairs become the recurrence coefficients d = 1 − a_t and b_t = √(1−a_t²)·i_t·u_t
        // (d in fp16, b_t in bf16, in the same packed places): the recurrence is then
        // h_t = (1 − d)·h_{t−1} + b_t. d ∈ [0, 1] keeps fp16's 11 significant bits; b_t scales
        // with u_t, so it takes bf16's float32 exponent range (any |u_t| a bf16 u can hold).
        float* sPar = reinterpret_cast<float*>(smem + S * k2StageBytes) + acc * 3 * 128;
        const int chalf = (warp - 2) / 4;  // which 64 of the 128 channels this warp forms
        named_bar_sync(1, 32 * epi_warps_of<EPI>());  // this CTA's epilogue warps: sPar is written
        uint16_t* out = reinterpret_cast<uint16_t*>(ep.C) + row * ep.ldc + (int64_t)n_blk * BN;  // 16-bit words
        // 4 chunks of 16 channels; the next chunk's TMEM load is in flight while one is formed
        uint32_t ra[2][16], rx[2][16];
        tmem_ld_x16(t_row + chalf * 64, ra[0]);
        tmem_ld_x16(t_row + 128 + chalf * 64, rx[0]);
        tmem_ld_wait16(ra[0], rx[0]);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int cur = k & 1;
          if (k + 1 < 4) {
            tmem_ld_x16(t_row + chalf * 64 + (k + 1) * 16, ra[cur ^ 1]);
            tmem_ld_x16(t_row + 128 + chalf * 64 + (k + 1) * 16, rx[cur ^ 1]);
          }
          const int c0 = chalf * 64 + k * 16;
          const uint32_t uw[8] = {uq[2 * k].x, uq[2 * k].y, uq[2 * k].z, uq[2 * k].w,
                                  uq[2 * k + 1].x, uq[2 * k + 1].y, uq[2 * k + 1].z, uq[2 * k + 1].w};
          uint32_t dh[8], mh[8], zah[8], zxh[8];
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const int c = c0 + j;
            const float2 u2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uw[j / 2]));
            const float2 za =
                make_float2(__uint_as_float(ra[cur][j]) + sPar[c], __uint_as_float(ra[cur][j + 1]) + sPar[c + 1]);
            const float2 zx = make_float2(__uint_as_float(rx[cur][j]) + sPar[128 + c],
                                          __uint_as_float(rx[cur][j + 1]) + sPar[128 + c + 1]);
            zah[j / 2] = pack_bf16x2(za.x, za.y);
            zxh[j / 2] = pack_bf16x2(zx.x, zx.y);
            float2 d, m;
            gate_fast2_pair(za, zx, make_float2(sPar[256 + c], sPar[256 + c + 1]), u2, d, m);
            const __half2 dd = __floats2half2_rn(d.x, d.y);
            const __nv_bfloat162 mm = __floats2bfloat162_rn(m.x, m.y);
            dh[j / 2] = *reinterpret_cast<const uint32_t*>(&dd);
            mh[j / 2] = *reinterpret_cast<const uint32_t*>(&mm);
          }
          if (row_ok) {
            uint4* pd = reinterpret_cast<uint4*>(out + c0);
            uint4* pm = reinterpret_cast<uint4*>(out + 128 + c0);
            pd[0] = make_uint4(dh[0], dh[1], dh[2], dh[3]);
            pd[1] = make_uint4(dh[4], dh[5], dh[6], dh[7]);
            pm[0] = make_uint4(mh[0], mh[1], mh[2], mh[3]);
            pm[1] = make_uint4(mh[4], mh[5], mh[6], mh[7]);
            if (ep.z_out != nullptr) {  // the pre-activations, saved for the backward
              uint4* za4 = reinterpret_cast<uint4*>(ep.z_out + row * ep.ldc + (int64_t)n_blk * BN + c0);
              uint4* zx4 = reinterpret_cast<uint4*>(ep.z_out + row * ep.ldc + (int64_t)n_blk * BN + 128 + c0);
              za4[0] = make_uint4(zah[0], zah[1], zah[2], zah[3]);
              za4[1] = make_uint4(zah[4], zah[5], zah[6], zah[7]);
              zx4[0] = make_uint4(zxh[0], zxh[1], zxh[2], zxh[3]);
              zx4[1] = make_uint4(zxh[4], zxh[5], zxh[6], zxh[7]);
            }
          }
          if (k + 1 < 4) tmem_ld_wait16(ra[cur ^ 1], rx[cur ^ 1]);
        }
      } else {
#pragma unroll 1
      for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_row + cc * 32, r);
        tmem_ld_wait();
        float v[32];
        const int col0 = cc * 32;
        if constexpr (EPI == EPI_GATES) {
          const int half = col0 / 128;
          const int ch0 = n_blk * 128 + (col0 % 128);
          const float* bias = half ? ep.b_x : ep.b_a;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int ch = ch0 + j;
            v[j] = __uint_as_float(r[j]) + (ch < ep.R ? __ldg(bias + ch) : 0.0f);
          }
          if (row_ok) store_row_bf16(ep.C + row * ep.ldc + (int64_t)n_blk * BN + col0, v);
        } else if constexpr (EPI == EPI_STORE_F32) {
          // float32 rows (N a multiple of 4): eight 16-byte stores per 32 columns
          const int gcol = n_blk * BN + col0;
          if (row_ok) {
            float4* d = reinterpret_cast<float4*>(ep.Cf + split_off + row * ep.ldc + gcol);
            float4 c[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
              c[q] = (ep.accumulate && gcol + 4 * q < ep.N) ? d[q] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              if (gcol + 4 * q < ep.N)
                d[q] = ep.accumulate
                           ? make_float4(c[q].x + __uint_as_float(r[4 * q]), c[q].y + __uint_as_float(r[4 * q + 1]),
                                         c[q].z + __uint_as_float(r[4 * q + 2]), c[q].w + __uint_as_float(r[4 * q + 3]))
                           : make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                         __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
          const int gcol = n_blk * BN + col0;
          if (row_ok) {
            if (gcol + 32 <= ep.N) {
              store_row_bf16(ep.C + row * ep.ldc + gcol, v);
            } else {
              uint4* d = reinterpret_cast<uint4*>(ep.C + row * ep.ldc + gcol);
#pragma unroll
              for (int q = 0; q < 4; ++q)
                if (gcol + 8 * q < ep.N)
                  d[q] = make_uint4(pack_bf16x2(v[8 * q + 0], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                                    pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
            }
          }
        }
      }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(leader_tempty0 + acc * 8);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
  } else {
    // ---------------- fused RG-LRU scan epilogue (both CTAs) ----------------
    // "Griffin：将门控线性循环与局部注意力混合以实现高效的语言模型", §实门线性循环单元 (RG-LRU),
    // Eq. (1)–(4). The CTA's 128 accumulator rows are 128 consecutive steps of one batch row
    // (T is a multiple of 128), its 256 columns z_a and z_x of 128 channels. Eight warps, as
    // in the coefficient epilogue: warp w holds rows 32·(w mod 4) … (TMEM lane quarter) and
    // one half of the channels; each thread is one step (row) and forms, for 16 channels at
    // a time, a_t = 1 − d and b_t = √(1−a_t²)·i_t·u_t (float32, never stored). The step's
    // affine maps h ↦ a_t h + b_t are composed across the warp's 32 rows through a small
    // shared-memory transpose (lane = channel and half of the rows, 16 steps in order):
    //   pass 1: each warp's map per channel; the four quarters' maps make
    //           the 128-step chunk's map; 128 threads (one per channel) publish it as the
    //           chunk's aggregate, take the incoming state from decoupled look-back over
    //           the earlier chunks of the same (batch row, channel block) (windows of 8,
    //           bounded waits), publish the inclusive state and hand each quarter its
    //           incoming state;
    //   pass 2: the same coefficients again (TMEM is read twice; the arithmetic is the
    //           same, so are the bits), the replay of each channel's 32 steps from the
    //           quarter's incoming state, and h_t = y_t back to the row's thread.
    // The pre-activations and coefficients never leave the SM. Forward progress: a chunk
    // waits only for earlier chunks, which are earlier tiles of the persistent grid (or the
    // other CTA of its own pair).
    const int quarter = warp & 3;
    const int chalf = (warp - 2) / 4;          // which 64 of the tile's 128 channels
    const int row_in_tile = quarter * 32 + lane;
    const int et = row_in_tile;                // channel of the look-back threads (chalf 0)
    uint8_t* escr = smem + S * k2StageBytes;
    float* sParAll = reinterpret_cast<float*>(escr);                    // [2 acc][3][128]
    float2* sQ = reinterpret_cast<float2*>(escr + kScanParBytes);       // [4 quarters][128]
    float* sS = reinterpret_cast<float*>(escr + kScanParBytes + 4 * 128 * 8);  // [4][128]
    float2* sT = reinterpret_cast<float2*>(escr + kScanParBytes + 4 * 128 * 8 + 4 * 128 * 4) +
                 (warp - 2) * 32 * kScanTPitch;  // this warp's [32 rows][17]
    const uint32_t leader_tempty0 = mapa_rank(smem_u32(&tempty_bar[0]), 0);
    const int R = ep.R;
    constexpr int kNT = 32 * epi_warps_of<EPI>();
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = cluster; tile < num_tiles; tile += n_clusters) {
      const int m_pair = tile / n_tiles_n, n_blk = tile % n_tiles_n;
      const int64_t m0 = (int64_t)m_pair * 256 + rank * 128;
      const bool cta_rows = m0 < M;  // (M is a multiple of 128: all 128 rows or none)
      const int64_t row = m0 + row_in_tile;
      // this thread's 64 values of u (its row, its half of the channels), before the
      // accumulator is ready; 8 channels are all valid or all not (R % 8 = 0)
      uint4 uq[8];
      {
        const int ch0 = n_blk * 128 + chalf * 64;
        const __nv_bfloat16* urow = ep.ub + row * R + ch0;
#pragma unroll
        for (int q8 = 0; q8 < 8; ++q8)
          uq[q8] = (cta_rows && ch0 + 8 * q8 < R) ? __ldg(reinterpret_cast<const uint4*>(urow) + q8)
                                                  : make_uint4(0u, 0u, 0u, 0u);
      }
      // the tile's channel parameters, also before the accumulator is ready (this parity's
      // buffer was last read by the tile two back, which every warp has finished)
      float* sPar = sParAll + acc * 3 * 128;
      if (chalf == 0) {
        const int ch = n_blk * 128 + et;
        const bool ok = ch < R;
        sPar[et] = ok ? __ldg(ep.b_a + ch) : 0.0f;
        sPar[128 + et] = ok ? __ldg(ep.b_x + ch) : 0.0f;
        sPar[256 + et] = ok ? decay_log_coeff(__ldg(ep.Lambda + ch)) : 0.0f;
      }
      if (!mbar_wait(&tfull_bar[acc], acc_phase, &abort_s)) {
        abort_s = 1;
        atomicOr(status, kStatusTimeout);
        break;
      }
      tc_fence_after();
      if (cta_rows) {
        const uint32_t t_row = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * BN;
        named_bar_sync(1, kNT);
        // (a_t, b_t) of this row for channels c0 … c0+15 of the tile
        auto coeffs = [&](int k, const uint32_t (&ra)[16], const uint32_t (&rx)[16], float (&A)[16],
                          float (&Bv)[16]) {
          const int c0 = chalf * 64 + k * 16;
          const uint32_t uw[8] = {uq[2 * k].x, uq[2 * k].y, uq[2 * k].z, uq[2 * k].w,
                                  uq[2 * k + 1].x, uq[2 * k + 1].y, uq[2 * k + 1].z, uq[2 * k + 1].w};
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const int c = c0 + j;
            const float2 u2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uw[j / 2]));
            const float2 za = make_float2(__uint_as_float(ra[j]) + sPar[c], __uint_as_float(ra[j + 1]) + sPar[c + 1]);
            const float2 zx = make_float2(__uint_as_float(rx[j]) + sPar[128 + c],
                                          __uint_as_float(rx[j + 1]) + sPar[128 + c + 1]);
            float2 d, m;
            gate_fast2_pair(za, zx, make_float2(sPar[256 + c], sPar[256 + c + 1]), u2, d, m);
            A[j] = 1.0f - d.x;
            A[j + 1] = 1.0f - d.y;
            Bv[j] = m.x;
            Bv[j + 1] = m.y;
          }
        };
        // ---- pass 1: each warp's map per channel → sQ[quarter][channel]
        {
          uint32_t ra[2][16], rx[2][16];
          tmem_ld_x16(t_row + chalf * 64, ra[0]);
          tmem_ld_x16(t_row + 128 + chalf * 64, rx[0]);
          tmem_ld_wait16(ra[0], rx[0]);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int cur = k & 1;
            if (k + 1 < 4) {
              tmem_ld_x16(t_row + chalf * 64 + (k + 1) * 16, ra[cur ^ 1]);
              tmem_ld_x16(t_row + 128 + chalf * 64 + (k + 1) * 16, rx[cur ^ 1]);
            }
            {
              float A[16], Bv[16];
              coeffs(k, ra[cur], rx[cur], A, Bv);
#pragma unroll
              for (int j = 0; j < 16; ++j) sT[lane * kScanTPitch + j] = make_float2(A[j], Bv[j]);
            }
            __syncwarp();
            // the transpose: lane (c, half) folds channel c over rows 16·half … 16·half + 15,
            // then the halves meet in one shuffle
            {
              const int c = lane & 15, r0 = (lane >> 4) * 16;
              float fa = 1.0f, fb = 0.0f;
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float2 m = sT[(r0 + i) * kScanTPitch + c];
                fb = fmaf(m.x, fb, m.y);
                fa *= m.x;
              }
              const float a2 = __shfl_down_sync(0xffffffffu, fa, 16);
              const float b2 = __shfl_down_sync(0xffffffffu, fb, 16);
              if (lane < 16) sQ[quarter * 128 + chalf * 64 + k * 16 + c] = make_float2(a2 * fa, fmaf(a2, fb, b2));
            }
            __syncwarp();
            if (k + 1 < 4) tmem_ld_wait16(ra[cur ^ 1], rx[cur ^ 1]);
          }
        }
        named_bar_sync(1, kNT);
        // ---- look-back: one thread per channel
        if (chalf == 0) {
          const int b_row = (int)(m0 / ep.T);
          const int chunk = (int)((m0 - (int64_t)b_row * ep.T) / 128);
          const int ch = n_blk * 128 + et;
          const bool cvalid = ch < R;
          float At = 1.0f, Bt = 0.0f;
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            const float2 mq = sQ[qq * 128 + et];
            Bt = fmaf(mq.x, Bt, mq.y);
            At *= mq.x;
          }
          const int64_t slot = (((int64_t)b_row * n_tiles_n + n_blk) * ep.n_chunks + chunk) * 128 + et;
          float hin;
          if (chunk == 0) {
            hin = (ep.h0 != nullptr && cvalid) ? ep.h0[(int64_t)b_row * R + ch] : 0.0f;
          } else {
            st_relaxed_u64g(ep.carry_agg + slot, ((uint64_t)__float_as_uint(Bt) << 32) | enc_carry(At));
            // the predecessors chunk − 1, chunk − 2, … in windows of 8: the nearest published
            // inclusive state, then the aggregates in front of it, oldest first
            float fA = 1.0f, fB = 0.0f;  // composed map of the predecessors already passed
            int d0 = 1;                  // depth of the window's first predecessor
            long long tw = 0;
            bool done = false;
            while (!done) {
              uint32_t wi[8];
              uint64_t ga[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const bool in = d0 + i <= chunk;
                wi[i] = in ? ld_relaxed_u32g(ep.carry_incl + slot - (int64_t)(d0 + i) * 128) : 0u;
                ga[i] = in ? ld_relaxed_u64g(ep.carry_agg + slot - (int64_t)(d0 + i) * 128) : 0ull;
              }
              int found = -1, have = 0;  // nearest inclusive; aggregates present in front of it
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                if (found < 0 && wi[i] != 0u) found = i;
                if (found < 0 && have == i && (uint32_t)ga[i] != 0u) have = i + 1;
              }
              if (found >= 0 && have >= found) {
                float h = 0.0f;
#pragma unroll
                for (int i = 0; i < 8; ++i)
                  if (i == found) h = dec_carry(wi[i]);
#pragma unroll
                for (int i = 7; i >= 0; --i)
                  if (i < found) h = fmaf(dec_carry((uint32_t)ga[i]), h, __uint_as_float((uint32_t)(ga[i] >> 32)));
                hin = fmaf(fA, h, fB);
                done = true;
              } else if (found < 0 && have == 8) {
                // the whole window is aggregates: fold it (newest first is the outer map)
                float wA = 1.0f, wB = 0.0f;
#pragma unroll
                for (int i = 7; i >= 0; --i) {
                  wB = fmaf(dec_carry((uint32_t)ga[i]), wB, __uint_as_float((uint32_t)(ga[i] >> 32)));
                  wA *= dec_carry((uint32_t)ga[i]);
                }
                fB = fmaf(fA, wB, fB);
                fA *= wA;
                d0 += 8;
              } else if (tw == 0) {
                tw = clock64();
              } else if (clock64() - tw > kWaitCycles) {
                atomicOr(status, kStatusTimeout);
                hin = fB;
                done = true;
              }
            }
          }
          const float hout = fmaf(At, hin, Bt);
          st_relaxed_u32g(ep.carry_incl + slot, enc_carry(hout));
          if (chunk == ep.n_chunks - 1 && ep.hT != nullptr && cvalid) ep.hT[(int64_t)b_row * R + ch] = hout;
          float sq = hin;
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            sS[qq * 128 + et] = sq;
            const float2 mq = sQ[qq * 128 + et];
            sq = fmaf(mq.x, sq, mq.y);
          }
        }
        named_bar_sync(1, kNT);
        // ---- pass 2: the same coefficients, the quarter's incoming state, h_t by scan
        {
          uint32_t ra[2][16], rx[2][16];
          tmem_ld_x16(t_row + chalf * 64, ra[0]);
          tmem_ld_x16(t_row + 128 + chalf * 64, rx[0]);
          tmem_ld_wait16(ra[0], rx[0]);
          __nv_bfloat16* yrow = ep.y + row * R + n_blk * 128;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int cur = k & 1;
            if (k + 1 < 4) {
              tmem_ld_x16(t_row + chalf * 64 + (k + 1) * 16, ra[cur ^ 1]);
              tmem_ld_x16(t_row + 128 + chalf * 64 + (k + 1) * 16, rx[cur ^ 1]);
            }
            const int c0 = chalf * 64 + k * 16;
            {
              float A[16], Bv[16];
              coeffs(k, ra[cur], rx[cur], A, Bv);
#pragma unroll
              for (int j = 0; j < 16; ++j) sT[lane * kScanTPitch + j] = make_float2(A[j], Bv[j]);
            }
            __syncwarp();
            // lane (c, half): its 16 steps of channel c; the second half starts from the first
            // half's map applied to the quarter's incoming state; then the replay, whose
            // states go back over the coefficients
            {
              const int c = lane & 15, r0 = (lane >> 4) * 16;
              float2 m[16];
              float fa = 1.0f, fb = 0.0f;
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                m[i] = sT[(r0 + i) * kScanTPitch + c];
                fb = fmaf(m[i].x, fb, m[i].y);
                fa *= m[i].x;
              }
              const float a2 = __shfl_up_sync(0xffffffffu, fa, 16);
              const float b2 = __shfl_up_sync(0xffffffffu, fb, 16);
              const float s0 = sS[quarter * 128 + c0 + c];
              float h = lane < 16 ? s0 : fmaf(a2, s0, b2);
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                h = fmaf(m[i].x, h, m[i].y);
                sT[(r0 + i) * kScanTPitch + c].x = h;
              }
            }
            __syncwarp();
            float Bv[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) Bv[j] = sT[lane * kScanTPitch + j].x;
            __syncwarp();
            if (n_blk * 128 + c0 < R) {  // 16 channels all valid or all not (R % 8 = 0, c0 % 16 = 0)
              uint4* py = reinterpret_cast<uint4*>(yrow + c0);
              py[0] = make_uint4(pack_bf16x2(Bv[0], Bv[1]), pack_bf16x2(Bv[2], Bv[3]), pack_bf16x2(Bv[4], Bv[5]),
                                 pack_bf16x2(Bv[6], Bv[7]));
              if (n_blk * 128 + c0 + 8 < R)
                py[1] = make_uint4(pack_bf16x2(Bv[8], Bv[9]), pack_bf16x2(Bv[10], Bv[11]),
                                   pack_bf16x2(Bv[12], Bv[13]), pack_bf16x2(Bv[14], Bv[15]));
            }
            if (k + 1 < 4) tmem_ld_wait16(ra[cur ^ 1], rx[cur ^ 1]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(leader_tempty0 + acc * 8);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer's shared memory stays valid until the leader's MMAs are done
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(k2TmemCols)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------------------
// Decode step GEMM, transposed and split over K inside a 4-CTA cluster.
// "Griffin：将门控线性循环与局部注意力混合以实现高效的语言模型", §实门线性循环单元 (RG-LRU),
// Eq. (1)–(4), one token: z = u_t · [W_a | W_x]ᵀ + b, then h ← a_t h + √(1−a_t²) i u_t, y = h.
// The weights are the large operand, so they are the MMA's M side and every weight row is
// read once per step. A cluster owns 128 channels. It holds two CTA pairs (cluster ranks
// 0–1 and 2–3), one per half of K; each pair runs 2-SM MMAs (cta_group::2, M = 256,
// N = 256): each CTA of a pair stages 64 rows of W_a and the same 64 rows of W_x, and 128 of
// the 256 batch rows. The two K halves then meet in shared memory: each CTA writes the
// partial sums of the batch half it does not own into its K-partner's shared memory
// (distributed shared memory, between two cluster barriers), adds the partner's, and
// applies the state update to its 64 channels × 128 batch rows with all its warps.
struct StepArgs {
  const float* b_a;
  const float* b_x;
  const float* u;        // u_t [B][R] float32
  float* h;              // [B][R], in place
  __nv_bfloat16* y;      // [B][R]
  const float* cla;      // [R]
  int B, R;
};
constexpr int kStepStages = 6;
constexpr int kStepABytes = 128 * BK * 2;  // 64 rows of W_a + the same 64 rows of W_x
constexpr int kStepBBytes = 128 * BK * 2;  // this CTA's 128 batch rows of u_t
constexpr int kStepStageBytes = kStepABytes + kStepBBytes;
constexpr int kStepRecvPitch = 132;  // floats per exchanged row (keeps 16-byte reads conflict-free)
constexpr int kStepXBytes = 128 * kStepRecvPitch * 4;  // one exchanged half: 128 rows
// after the mainloop: zs [0, 64 KB), the half received [64 KB, +kStepXBytes), the half sent after it
constexpr int kStepSmem = 65536 + 2 * kStepXBytes + 1024;
constexpr int kStepTmemCols = 256;
constexpr int kStepHalf = 128 * 128;  // floats: 128 accumulator rows × 128 batch columns
// warps: 0 TMA, 1 MMA, 2–9 TMEM readers (warp w reads lane quarter w % 4, column half
// (w − 2) / 4), all twelve for the state update
constexpr int kStepThreads = 384;
static_assert(kStepStages * kStepStageBytes + 1024 <= kStepSmem, "the ring fits");
static_assert(kStepSmem <= 227 * 1024, "shared memory");

// Bulk copy of `bytes` from this CTA's shared memory to another CTA's (cluster addresses for
// the destination and its mbarrier), completing on that mbarrier.
__device__ __forceinline__ void bulk_copy_to_cta(uint32_t dst_cluster, const void* src, uint32_t bytes,
                                                 uint32_t mbar_cluster) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   dst_cluster),
               "r"(smem_u32(src)), "r"(bytes), "r"(mbar_cluster)
               : "memory");
}
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar, uint16_t mask) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                   smem_u32(bar)),
               "h"(mask)
               : "memory");
}

__global__ void __launch_bounds__(kStepThreads, 1)
    step_kernel(const __grid_constant__ CUtensorMap tmWa, const __grid_constant__ CUtensorMap tmWx,
                const __grid_constant__ CUtensorMap tmU, StepArgs ep, unsigned* status) {
  constexpr int S = kStepStages;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[S];
  __shared__ __align__(8) uint64_t empty_bar[S];
  __shared__ __align__(8) uint64_t tfull_bar;
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ __align__(8) uint64_t xbar;  // the K-partner's half has landed
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t crank = cluster_ctarank();  // 0..3
  const uint32_t rank = crank & 1u;          // rank inside the CTA pair
  const uint32_t pair_leader = crank & 2u;   // cluster rank of this pair's leader
  const bool leader = rank == 0;
  const int kh = (int)(crank >> 1);          // K half, and the batch half this CTA updates
  const uint16_t pair_mask = (uint16_t)(0x3u << pair_leader);
  const int cblk = blockIdx.x / 4;           // 128-channel block
  const int Kh = ep.R / 2;
  const int k0 = kh * Kh;
  const int k_blocks = Kh / BK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    mbar_init(&tfull_bar, 1);
    mbar_init(&drain_bar, 1);
    mbar_init(&xbar, 1);
    abort_s = 0;
    fence_barrier_init();
    mbar_arrive_expect_tx(&xbar, kStepXBytes);
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmWa);
    tma_prefetch_desc(&tmWx);
    tma_prefetch_desc(&tmU);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_s)),
                 "r"(kStepTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync_all();  // every CTA's barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_s;
  const uint32_t leader_full0 = mapa_rank(smem_u32(&full_bar[0]), pair_leader);
  const int wrow = cblk * 128 + (int)rank * 64;
  const int pre = k_blocks < S ? k_blocks : S;  // stages whose weights load before u_t exists
  if (warp == 0) {
    // The weights do not depend on the decode conv kernel: while it runs, lane 0 fills the
    // first stages' weight halves (their u_t halves follow once u_t is written). (An L2
    // prefetch of the CTA's whole weight slice here as well made the step slower.)
    if (lane == 0) {
      for (int kb = 0; kb < pre; ++kb) {
        uint8_t* sa = smem + kb * kStepStageBytes;
        const uint32_t lbar = leader_full0 + kb * 8;
        if (leader) mbar_arrive_expect_tx(&full_bar[kb], 2 * kStepStageBytes);
        tma_load_2d_2sm(sa, &tmWa, lbar, k0 + kb * BK, wrow);
        tma_load_2d_2sm(sa + 64 * BK * 2, &tmWx, lbar, k0 + kb * BK, wrow);
      }
    }
  }
  // launched as a programmatic dependent of the decode conv kernel: everything above
  // overlapped it; u_t, u_t in float32 and c·log σ(Λ) are its results
  pdl_wait();

  // The state update's inputs do not depend on the GEMM: every thread loads its u_t and h
  // values now and holds them in registers through the mainloop. Thread t updates channel
  // j = t % 64 of this CTA's 64 and the batch columns c = t / 64 + kPhases·i of its half.
  constexpr int kPhases = kStepThreads / 64;
  constexpr int kPer = (128 + kPhases - 1) / kPhases;
  const int uj = threadIdx.x % 64;
  const int uch = cblk * 128 + (int)rank * 64 + uj;
  float uv[kPer], hv[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int c = (int)threadIdx.x / 64 + kPhases * i;
    const int b = kh * 128 + c;
    const int64_t idx = (int64_t)b * ep.R + uch;
    const bool ok = c < 128 && b < ep.B;
    uv[i] = ok ? __ldg(ep.u + idx) : 0.0f;
    hv[i] = ok ? ep.h[idx] : 0.0f;
  }
  const float ba = __ldg(ep.b_a + uch), bx = __ldg(ep.b_x + uch), cl = __ldg(ep.cla + uch);

  if (warp == 0) {
    // ---------------- TMA producer (every CTA) ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int kb = 0; kb < k_blocks; ++kb) {
        uint8_t* sa = smem + stage * kStepStageBytes;
        uint8_t* sb = sa + kStepABytes;
        const uint32_t lbar = leader_full0 + stage * 8;
        const int kc = k0 + kb * BK;
        if (kb >= pre) {  // the first `pre` stages hold their weights already
          if (!mbar_wait(&empty_bar[stage], phase ^ 1, &abort_s)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2 * kStepStageBytes);
          tma_load_2d_2sm(sa, &tmWa, lbar, kc, wrow);
          tma_load_2d_2sm(sa + 64 * BK * 2, &tmWx, lbar, kc, wrow);
        }
        tma_load_2d_2sm(sb, &tmU, lbar, kc, (int)rank * 128);
        if (++stage == S) { stage = 0; phase ^= 1; }
      }
      if (!ok) { abort_s = 1; atomicOr(status, kStatusTimeout); }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (pair leaders only) ----------------
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int kb = 0; kb < k_blocks; ++kb) {
        if (!mbar_wait(&full_bar[stage], phase, &abort_s)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + stage * kStepStageBytes);
        const uint32_t b_addr = a_addr + kStepABytes;
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)
          umma_f16_2sm(tmem_base, umma_desc_sw128(a_addr + k * 32), umma_desc_sw128(b_addr + k * 32), k2Idesc,
                       (kb | k) != 0 ? 1u : 0u);
        umma_commit_pair(&empty_bar[stage], pair_mask);
        if (++stage == S) { stage = 0; phase ^= 1; }
      }
      if (ok) umma_commit_pair(&tfull_bar, pair_mask);
      if (!ok) { abort_s = 1; atomicOr(status, kStatusTimeout); }
      asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                       smem_u32(&drain_bar))
                   : "memory");
      volatile int never = 0;
      (void)mbar_wait(&drain_bar, 0, &never);
    }
  }

  // ---------------- K-half exchange and state update (every CTA, every warp) ----------------
  const int q = warp & 3;          // TMEM lanes 32q … 32q+31
  const int row = q * 32 + lane;   // accumulator row: W_a row (row < 64) or W_x row
  const bool epi = warp >= 2 && warp < 10;  // TMEM readers
  const int chalf = (warp - 2) / 4;         // which 64 of a 128-column half this warp moves
  const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16);
  constexpr int kRecvPitch = kStepRecvPitch;
  float* zs = reinterpret_cast<float*>(smem);                                    // [128 batch cols][128 rows]
  float* recv = reinterpret_cast<float*>(smem + kStepHalf * 4);                  // [128 rows][kRecvPitch]
  float* sendb = reinterpret_cast<float*>(smem + kStepHalf * 4 + kStepXBytes);   // [128 rows][kRecvPitch]
  if (epi) {
    if (!mbar_wait(&tfull_bar, 0, &abort_s)) {
      abort_s = 1;
      atomicOr(status, kStatusTimeout);
    }
    tc_fence_after();
    // the partial sums of the batch half the K-partner updates, staged for the copy
    const int other = 1 - kh;
    float* out = sendb + row * kRecvPitch;
#pragma unroll 1
    for (int cc = 2 * chalf; cc < 2 * chalf + 2; ++cc) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(t_row + other * 128 + cc * 32, r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; j += 4)
        *reinterpret_cast<float4*>(out + cc * 32 + j) =
            make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]), __uint_as_float(r[j + 2]),
                        __uint_as_float(r[j + 3]));
    }
    fence_proxy_async_smem();  // the staged half is read by the bulk copy
  }
  tc_fence_before();
  cluster_sync_all();  // every MMA of the cluster is done (the rings are free) and the halves are staged
  tc_fence_after();
  if (threadIdx.x == 0) {
    // one bulk copy into the K-partner's receive buffer, completing on its mbarrier
    const uint32_t partner = crank ^ 2u;
    bulk_copy_to_cta(mapa_rank(smem_u32(recv), partner), sendb, kStepXBytes, mapa_rank(smem_u32(&xbar), partner));
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
  }
  if (epi) {
    if (!mbar_wait(&xbar, 0, &abort_s)) {
      abort_s = 1;
      atomicOr(status, kStatusTimeout);
    }
    // full sums of this CTA's batch half, staged as zs[batch column][accumulator row]
    const float* in = recv + row * kRecvPitch;
#pragma unroll 1
    for (int cc = 2 * chalf; cc < 2 * chalf + 2; ++cc) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(t_row + kh * 128 + cc * 32, r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        const float4 p = *reinterpret_cast<const float4*>(in + cc * 32 + j);
        zs[(cc * 32 + j + 0) * 128 + row] = __uint_as_float(r[j + 0]) + p.x;
        zs[(cc * 32 + j + 1) * 128 + row] = __uint_as_float(r[j + 1]) + p.y;
        zs[(cc * 32 + j + 2) * 128 + row] = __uint_as_float(r[j + 2]) + p.z;
        zs[(cc * 32 + j + 3) * 128 + row] = __uint_as_float(r[j + 3]) + p.w;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  {
    // h ← a_t h + √(1−a_t²) i u_t and y = h for 64 channels × 128 batch rows, by all twelve
    // warps, from the u_t and h values loaded at the start
    // two batch columns at a time, in packed f32x2 arithmetic (d = 1 − a_t, b_t)
    static_assert(kPer % 2 == 0, "columns in pairs");
#pragma unroll
    for (int i = 0; i < kPer; i += 2) {
      const int c0 = (int)threadIdx.x / 64 + kPhases * i;
      const int c1 = c0 + kPhases;
      const int c1r = c1 < 128 ? c1 : 127;  // (a column past the half is computed, not stored)
      float2 d, bt;
      gate_fast2_pair(make_float2(zs[c0 * 128 + uj] + ba, zs[c1r * 128 + uj] + ba),
                      make_float2(zs[c0 * 128 + 64 + uj] + bx, zs[c1r * 128 + 64 + uj] + bx), make_float2(cl, cl),
                      make_float2(uv[i], uv[i + 1]), d, bt);
      const float2 hn = __ffma2_rn(make_float2(1.0f - d.x, 1.0f - d.y), make_float2(hv[i], hv[i + 1]), bt);
      const int b0 = kh * 128 + c0, b1 = kh * 128 + c1;
      if (c0 < 128 && b0 < ep.B) {
        const int64_t idx = (int64_t)b0 * ep.R + uch;
        ep.h[idx] = hn.x;
        ep.y[idx] = __float2bfloat16_rn(hn.x);
      }
      if (c1 < 128 && b1 < ep.B) {
        const int64_t idx = (int64_t)b1 * ep.R + uch;
        ep.h[idx] = hn.y;
        ep.y[idx] = __float2bfloat16_rn(hn.y);
      }
    }
  }

  if (threadIdx.x == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kStepTmemCols)
                 : "memory");
  }
}

template <int EPI, bool DUAL>
cudaError_t launch_tc2(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, int64_t M, int K,
                       int n_tiles_n, const EpiArgs& ep, unsigned* status, cudaStream_t s) {
  auto kern = gemm2_kernel<EPI, DUAL>;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_of<EPI>());
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const int64_t m_pairs = (M + 255) / 256;
  const int64_t tiles = m_pairs * n_tiles_n * (ep.k_split > 1 ? ep.k_split : 1);
  if (tiles > INT32_MAX) return cudaErrorInvalidValue;
  const int clusters = (int)std::min<int64_t>(tiles, num_sms() / 2);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(threads_of<EPI>());
  cfg.dynamicSmemBytes = smem_of<EPI>();
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // the kernel waits (pdl_wait)
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, a, b0, b1, M, K, n_tiles_n, (int)tiles, ep, status);
}

// ---------------------------------------------------------------------------------------
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

bool make_map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                 uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn fn = get_encode_tiled();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN, int EPI, bool DUAL>
cudaError_t launch_tc(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, int64_t M, int K,
                      int n_tiles_n, const EpiArgs& ep, unsigned* status, cudaStream_t s) {
  using Cfg = GemmCfg<BN>;
  auto kern = gemm_tc_kernel<BN, EPI, DUAL>;
  static bool attr_set = false;  // per instantiation; benign race (idempotent)
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int64_t m_tiles = (M + BM - 1) / BM;
  const int64_t tiles = m_tiles * n_tiles_n;
  if (tiles > INT32_MAX) return cudaErrorInvalidValue;
  const int grid = (int)std::min<int64_t>(tiles, num_sms());
  kern<<<grid, kGemmThreads, Cfg::kSmem, s>>>(a, b0, b1, M, K, n_tiles_n, (int)tiles, ep, status);
  return cudaGetLastError();
}

}  // namespace

// Status word for GEMM launches that come without a workspace.
__device__ unsigned g_gemm_status;

EncodeTiledFn get_encode_tiled() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  return g_encode;
}

int num_sms() {
  static int n[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (n[dev] == 0) cudaDeviceGetAttribute(&n[dev], cudaDevAttrMultiProcessorCount, dev);
  return n[dev];
}

cudaError_t launch_gate_scan_bf16(const ScanFusedArgs& f, cudaStream_t s) {
  // 2-SM gate GEMM with the RG-LRU scan in its epilogue; needs T % 128 == 0.
  const int64_t M = (int64_t)f.B * f.T;
  CUtensorMap ma, mb0, mb1;
  if (!make_map_2d(&ma, f.u, f.R, M, (uint64_t)f.R * 2, BK, BM)) return cudaErrorInvalidValue;
  if (!make_map_2d(&mb0, f.W_a, f.R, f.R, (uint64_t)f.R * 2, BK, 128)) return cudaErrorInvalidValue;
  if (!make_map_2d(&mb1, f.W_x, f.R, f.R, (uint64_t)f.R * 2, BK, 128)) return cudaErrorInvalidValue;
  EpiArgs ep{};
  ep.b_a = f.b_a;
  ep.b_x = f.b_x;
  ep.R = f.R;
  ep.y = static_cast<__nv_bfloat16*>(f.y);
  ep.ub = static_cast<const __nv_bfloat16*>(f.u);
  ep.Lambda = f.Lambda;
  ep.h0 = f.h0;
  ep.hT = f.hT;
  ep.carry_agg = f.carry_agg;
  ep.carry_incl = f.carry_incl;
  ep.T = f.T;
  ep.n_chunks = f.T / 128;
  const int n_tiles_n = (f.R + 127) / 128;
  return launch_tc2<EPI_SCAN, true>(ma, mb0, mb1, M, f.R, n_tiles_n, ep, f.status, s);
}

unsigned* global_status_word() {
  static unsigned* p[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (p[dev] == nullptr) {
    unsigned* q = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&q), g_gemm_status) != cudaSuccess) return nullptr;
    p[dev] = q;
  }
  return p[dev];
}

cudaError_t launch_gemm_gates_bf16(const void* u, const void* Wa, const float* ba, const void* Wx, const float* bx,
                                   void* z, int64_t M, int R, unsigned* status, cudaStream_t s) {
  // 2-SM tiles: 256 tokens × 256 packed columns (128 channels × two gates); the leader
  // CTA stages 128 rows of W_a, its peer the same 128 rows of W_x.
  CUtensorMap ma, mb0, mb1;
  if (!make_map_2d(&ma, u, R, M, (uint64_t)R * 2, BK, BM)) return cudaErrorInvalidValue;
  if (!make_map_2d(&mb0, Wa, R, R, (uint64_t)R * 2, BK, 128)) return cudaErrorInvalidValue;
  if (!make_map_2d(&mb1, Wx, R, R, (uint64_t)R * 2, BK, 128)) return cudaErrorInvalidValue;
  EpiArgs ep{};
  ep.C = static_cast<__nv_bfloat16*>(z);
  ep.ldc = gate_pitch(R);
  ep.b_a = ba;
  ep.b_x = bx;
  ep.R = R;
  const int n_tiles_n = (R + 127) / 128;
  return launch_tc2<EPI_GATES, true>(ma, mb0, mb1, M, R, n_tiles_n, ep, status, s);
}

cudaError_t launch_gemm_coeffs_bf16(const void* u, const void* Wa, const float* ba, const void* Wx, const float* bx,
                                    const float* Lambda, void* g, int64_t M, int R, unsigned* status, cudaStream_t s,
                                    void* z_out) {
  // the gate GEMM's tiles, with the recurrence coefficients formed in the epilogue
  CUtensorMap ma, mb0, mb1;
  if (!make_map_2d(&ma, u, R, M, (uint64_t)R * 2, BK, BM)) return cudaErrorInvalidValue;
  if (!make_map_2d(&mb0, Wa, R, R, (uint64_t)R * 2, BK, 128)) return cudaErrorInvalidValue;
  if (!make_map_2d(&mb1, Wx, R, R, (uint64_t)R * 2, BK, 128)) return cudaErrorInvalidValue;
  EpiArgs ep{};
  ep.C = static_cast<__nv_bfloat16*>(g);
  ep.ldc = gate_pitch(R);
  ep.b_a = ba;
  ep.b_x = bx;
  ep.Lambda = Lambda;
  ep.R = R;
  ep.ub = static_cast<const __nv_bfloat16*>(u);
  ep.z_out = static_cast<__nv_bfloat16*>(z_out);
  const int n_tiles_n = (R + 127) / 128;
  return launch_tc2<EPI_COEF, true>(ma, mb0, mb1, M, R, n_tiles_n, ep, status, s);
}

cudaError_t launch_gemm_bf16(const void* A, const void* Bm, void* C, int64_t M, int N, int K, int64_t ldc,
                             unsigned* status, cudaStream_t s) {
  // 2-SM tiles 256 × 256: each CTA of the pair stages 128 rows of A and 128 rows of B.
  CUtensorMap ma, mb;
  if (!make_map_2d(&ma, A, K, M, (uint64_t)K * 2, BK, BM)) return cudaErrorInvalidValue;
  if (!make_map_2d(&mb, Bm, K, N, (uint64_t)K * 2, BK, 128)) return cudaErrorInvalidValue;
  EpiArgs ep{};
  ep.C = static_cast<__nv_bfloat16*>(C);
  ep.ldc = ldc;
  ep.N = N;
  const int n_tiles_n = (N + 255) / 256;
  return launch_tc2<EPI_STORE, false>(ma, mb, mb, M, K, n_tiles_n, ep, status, s);
}

cudaError_t launch_gemm_f32out(const void* A, const void* Bm, float* C, int64_t M, int N, int K, int64_t ldc,
                               bool accumulate, unsigned* status, cudaStream_t s) {
  // as launch_gemm_bf16, with float32 output rows (added to C's when `accumulate`)
  CUtensorMap ma, mb;
  if (!make_map_2d(&ma, A, K, M, (uint64_t)K * 2, BK, BM)) return cudaErrorInvalidValue;
  if (!make_map_2d(&mb, Bm, K, N, (uint64_t)K * 2, BK, 128)) return cudaErrorInvalidValue;
  EpiArgs ep{};
  ep.Cf = C;
  ep.ldc = ldc;
  ep.N = N;
  ep.accumulate = accumulate ? 1 : 0;
  const int n_tiles_n = (N + 255) / 256;
  return launch_tc2<EPI_STORE_F32, false>(ma, mb, mb, M, K, n_tiles_n, ep, status, s);
}

cudaError_t launch_gemm_f32out_mn(const void* A, int64_t lda, const void* Bm, int64_t ldb, float* C, int M, int N,
                                  int64_t K, int64_t ldc, unsigned* status, cudaStream_t s) {
  // C = Aᵀ B over K rows: A [K][lda] holding M columns, B [K][ldb] holding N columns, both
  // staged MN-major (no transposed copies); rows past K read as zeros
  if (lda % 8 || ldb % 8 || (reinterpret_cast<uintptr_t>(A) & 15) || (reinterpret_cast<uintptr_t>(Bm) & 15) ||
      K > INT32_MAX)
    return cudaErrorInvalidValue;
  CUtensorMap ma, mb;
  if (!make_map_2d(&ma, A, M, K, (uint64_t)lda * 2, 64, BK)) return cudaErrorInvalidValue;
  if (!make_map_2d(&mb, Bm, N, K, (uint64_t)ldb * 2, 64, BK)) return cudaErrorInvalidValue;
  EpiArgs ep{};
  ep.Cf = C;
  ep.ldc = ldc;
  ep.N = N;
  ep.a_mn = 1;
  ep.b_mn = 1;
  const int n_tiles_n = (N + 255) / 256;
  return launch_tc2<EPI_STORE_F32, false>(ma, mb, mb, M, (int)K, n_tiles_n, ep, status, s);
}

cudaError_t launch_gemm_f32out_wcat(const void* A, const void* W0, const void* W1, float* C, int64_t M, int N,
                                    int Kh, int64_t ldc, bool accumulate, unsigned* status, cudaStream_t s) {
  // C (+)= A·[W0; W1]: A [M][2Kh] K-major, W0 and W1 [Kh][N] row-major read in place as the
  // MN-major B operand, W0 for the k-blocks below Kh and W1 above (Kh a multiple of BK)
  if (Kh % BK || N % 8) return cudaErrorInvalidValue;
  CUtensorMap ma, mb0, mb1;
  if (!make_map_2d(&ma, A, 2 * (uint64_t)Kh, M, (uint64_t)Kh * 4, BK, BM)) return cudaErrorInvalidValue;
  if (!make_map_2d(&mb0, W0, N, Kh, (uint64_t)N * 2, 64, BK)) return cudaErrorInvalidValue;
  if (!make_map_2d(&mb1, W1, N, Kh, (uint64_t)N * 2, 64, BK)) return cudaErrorInvalidValue;
  EpiArgs ep{};
  ep.Cf = C;
  ep.ldc = ldc;
  ep.N = N;
  ep.accumulate = accumulate ? 1 : 0;
  ep.b_mn = 1;
  ep.b_split_k = Kh;
  const int n_tiles_n = (N + 255) / 256;
  return launch_tc2<EPI_STORE_F32, false>(ma, mb0, mb1, M, 2 * Kh, n_tiles_n, ep, status, s);
}

namespace {
// out[m][0 … N) = bf16(Σ_s part[s][m][·]) for partial sums part [S][M][N] float32, N % 8 == 0.
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float* __restrict__ part, int S, int64_t M, int N,
                                                          int64_t ldc, __nv_bfloat16* __restrict__ out) {
  pdl_wait();  // the partial sums are the GEMM's output
  pdl_launch_dependents();
  const int64_t n8 = N / 8;
  const int64_t total = M * n8;
  const int64_t stride = M * (int64_t)N;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t m = i / n8, c = (i - m * n8) * 8;
    float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int sl = 0; sl < S; ++sl) {
      const float4* p = reinterpret_cast<const float4*>(part + sl * stride + m * N + c);
      const float4 a = __ldcs(p), b = __ldcs(p + 1);
      v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
      v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
    }
    *reinterpret_cast<uint4*>(out + m * ldc + c) =
        make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
  }
}
}  // namespace

int skinny_splits(int64_t M, int N, int K, size_t part_bytes) {
  // Few output tiles (M = a decode batch): split K so that about every SM pair works, at
  // least 4 k-blocks a slice, the slices' float32 partial sums within part_bytes; no empty
  // slice.
  const int64_t m_pairs = (M + 255) / 256;
  const int n_tiles_n = (N + 255) / 256;
  const int k_blocks = (K + BK - 1) / BK;
  const int64_t tiles = m_pairs * n_tiles_n;
  const int clusters = num_sms() / 2;
  int ksp = 1;
  if (part_bytes > 0 && tiles * 2 <= clusters && N % 8 == 0) {
    ksp = (int)std::min<int64_t>(clusters / tiles, k_blocks / 4);
    while (ksp > 1 && (size_t)ksp * M * N * 4 > part_bytes) --ksp;
  }
  if (ksp <= 1) return 1;
  const int kb_per = (k_blocks + ksp - 1) / ksp;
  return (k_blocks + kb_per - 1) / kb_per;
}

cudaError_t launch_gemm_partials(const void* A, const void* Bm, int64_t M, int N, int K, float* part, int ksp,
                                 unsigned* status, cudaStream_t s) {
  const int k_blocks = (K + BK - 1) / BK;
  const int kb_per = (k_blocks + ksp - 1) / ksp;
  if (ksp < 1 || (k_blocks + kb_per - 1) / kb_per != ksp) return cudaErrorInvalidValue;
  CUtensorMap ma, mb;
  if (!make_map_2d(&ma, A, K, M, (uint64_t)K * 2, BK, BM)) return cudaErrorInvalidValue;
  if (!make_map_2d(&mb, Bm, K, N, (uint64_t)K * 2, BK, 128)) return cudaErrorInvalidValue;
  EpiArgs ep{};
  ep.Cf = part;
  ep.ldc = N;
  ep.N = N;
  ep.k_split = ksp;
  ep.kb_per = kb_per;
  ep.split_stride = M * (int64_t)N;
  return launch_tc2<EPI_STORE_F32, false>(ma, mb, mb, M, K, (N + 255) / 256, ep, status, s);
}

cudaError_t launch_gemm_bf16_skinny(const void* A, const void* Bm, void* C, int64_t M, int N, int K, int64_t ldc,
                                    float* part, size_t part_bytes, unsigned* status, cudaStream_t s) {
  // the slices' partial sums, then one kernel summing them into bf16
  const int ksp = part != nullptr ? skinny_splits(M, N, K, part_bytes) : 1;
  if (ksp <= 1) return launch_gemm_bf16(A, Bm, C, M, N, K, ldc, status, s);
  cudaError_t e = launch_gemm_partials(A, Bm, M, N, K, part, ksp, status, s);
  if (e != cudaSuccess) return e;
  const int64_t work = M * (N / 8);
  const int blocks = (int)std::min<int64_t>((work + 255) / 256, (int64_t)num_sms() * 8);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, splitk_reduce_kernel, (const float*)part, ksp, M, N, ldc,
                            static_cast<__nv_bfloat16*>(C));
}

namespace {
// Whether the cluster step kernel covers (B, R) on the current device.
bool step_cluster_usable(int B, int R) {
  if (B > 256 || R % 128 != 0) return false;
  static int ok[64] = {0};  // 0 unknown, 1 usable, -1 not
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (ok[dev] == 0) {
    ok[dev] = -1;
    if (cudaFuncSetAttribute(step_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kStepSmem) == cudaSuccess &&
        cudaFuncSetAttribute(step_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 0) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(4);
      cfg.blockDim = dim3(kStepThreads);
      cfg.dynamicSmemBytes = kStepSmem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 4;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, step_kernel, &cfg) == cudaSuccess && n >= 1) ok[dev] = 1;
    }
    (void)cudaGetLastError();
  }
  return ok[dev] == 1;
}
}  // namespace

cudaError_t launch_gemm_step_bf16(const void* u_t, const float* u_f32, const void* Wa, const float* ba,
                                  const void* Wx, const float* bx, const float* cla, float* h, void* y_t, int B,
                                  int R, unsigned* status, cudaStream_t s) {
  if (step_cluster_usable(B, R)) {
    CUtensorMap mwa, mwx, mu;
    if (!make_map_2d(&mwa, Wa, R, R, (uint64_t)R * 2, BK, 64)) return cudaErrorInvalidValue;
    if (!make_map_2d(&mwx, Wx, R, R, (uint64_t)R * 2, BK, 64)) return cudaErrorInvalidValue;
    if (!make_map_2d(&mu, u_t, R, B, (uint64_t)R * 2, BK, 128)) return cudaErrorInvalidValue;
    StepArgs ep{};
    ep.b_a = ba;
    ep.b_x = bx;
    ep.u = u_f32;
    ep.h = h;
    ep.y = static_cast<__nv_bfloat16*>(y_t);
    ep.cla = cla;
    ep.B = B;
    ep.R = R;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(4 * (R / 128));
    cfg.blockDim = dim3(kStepThreads);
    cfg.dynamicSmemBytes = kStepSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 4;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // overlap the decode conv's tail
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, step_kernel, mwa, mwx, mu, ep, status);
  }
  constexpr int BN = 128;
  CUtensorMap ma, mb0, mb1;
  if (!make_map_2d(&ma, u_t, R, B, (uint64_t)R * 2, BK, BM)) return cudaErrorInvalidValue;
  if (!make_map_2d(&mb0, Wa, R, R, (uint64_t)R * 2, BK, BN / 2)) return cudaErrorInvalidValue;
  if (!make_map_2d(&mb1, Wx, R, R, (uint64_t)R * 2, BK, BN / 2)) return cudaErrorInvalidValue;
  EpiArgs ep{};
  ep.b_a = ba;
  ep.b_x = bx;
  ep.R = R;
  ep.u = u_f32;
  ep.h = h;
  ep.y = static_cast<__nv_bfloat16*>(y_t);
  ep.cla = cla;
  const int n_tiles_n = (R + BN / 2 - 1) / (BN / 2);
  return launch_tc<BN, EPI_STEP, true>(ma, mb0, mb1, B, R, n_tiles_n, ep, status, s);
}


}  // namespace rglru
