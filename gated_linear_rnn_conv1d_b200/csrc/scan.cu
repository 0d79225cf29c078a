// RG-LRU chunked scan, in two forms:
//  * from pre-activations: Conv1D recompute + σ gates + log-space decay + chunked diagonal
//    recurrence; one HBM read of x and of the packed gate pre-activations z, one write of y;
//  * from recurrence coefficients (bf16 IO): d = 1 − a_t (fp16) and b_t = √(1−a_t²)·i_t·u_t
//    (bf16), formed by the gate GEMM's epilogue; one HBM read of (d, b), one write of y.
//
// Math: "Griffin：将门控线性循环与局部注意力混合以实现高效的语言模型",
// §实门线性循环单元 (RG-LRU), Eq. (1)–(4); §循环块 for the Conv1D and the GeLU branch.
// Parallelisation: the recurrence h_t = a_t h_{t-1} + b_t is linear in h (neither gate
// reads h_{t-1}), so a run of steps composes into one affine map h ↦ A h + B, with
// (A₁,B₁) then (A₂,B₂) giving (A₂A₁, A₂B₁ + B₂). Runs are scanned independently and their
// summaries passed along ("Griffin's Compromise: Combining Gated Linear Recurrence with
// Local Attention", §Hawk, "Parallel scan").
//
// Tiles. A tile is one batch row b, CW consecutive channels (128 for bf16, 64 for f32)
// and kScanTC = 64 consecutive steps: 32 channel groups of V channels (4 bf16 or 2 f32)
// × 16 sub-chunks of 4 steps.
//
// One persistent CTA per SM takes tiles in order of a ticket (its first two fixed, the rest
// from an atomic counter) — time-chunk-major, so every tile a CTA waits for was taken
// earlier by a running CTA (forward progress) —
// and runs them through a software pipeline of three warp roles:
//   producer warp    takes tickets and, ahead of the compute warps, fills a ring of stages
//                    (3, or 5 for the smaller coefficient stages): TMA copies of the tile's
//                    x rows (with the 3-row conv halo; rows before t = 0 arrive as zeros),
//                    z_a and z_x, plus the tile's parameters (taps, conv bias, c·log σ(Λ))
//                    written into the stage — or only the two coefficient blocks — and the
//                    tile's decoded coordinates;
//   compute warps    (16, one per sub-chunk of 4 steps; lane = channel group; the
//                    coefficient form splits them into two groups of 8 on alternate tiles,
//                    one per sub-chunk of 8 steps), for tile k:
//     phase 1  recompute u in float32, apply the gates and the log-space decay (or read
//              the coefficients), fold the sub-chunk's 4 steps into an affine map
//              (float32); the pre-activation form writes the per-step replay values
//              (1 − a_t, b_t) over the z_a, z_x slots they came from;
//     phase 3  (of the group's previous tile, whose incoming states are ready by now)
//              replay the sub-chunk from its incoming state and write y, then release
//              the stage;
//   look-back warps  (groups of 2 warps, two channels per thread for bf16; the coefficient
//                    form has two groups taking alternate tiles) read the state entering
//                    tile k — the inclusive state its predecessor chunk publishes, or h0 —
//                    while phase 1 of tile k runs; once the sub-chunk maps are in, they
//                    compose them, publish the tile's inclusive state and hand every
//                    sub-chunk its incoming state. A published state is a self-validating
//                    word (an exact XOR encoding whose zero is never a published value, so
//                    zeroed memory reads as "not yet"): one relaxed load, no fence or flag.
// Every wait is bounded. Warps of different roles meet at mbarriers (stage full / empty,
// states ready) and at a named barrier (maps ready); map buffers, maps barriers and states
// barriers rotate with the tile number (mod 2, or mod 4 for two compute groups) so that
// none is reused before every role is done with it. The compute warps never wait for one
// another.
// The replay values of the pre-activation bf16 path are stored as bf16 (1 − a_t, b_t): their
// rounding only touches y inside one 4-step sub-chunk, while the published states and h_T
// come from the float32 maps. Of the coefficients, d ∈ [0, 1] is fp16 (11 significant bits:
// its relative error multiplies into every carried state) and b_t is bf16 (it scales with
// u_t, so it needs float32's exponent range); everything composed from them (maps, states,
// h_T) is float32.
#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "gate_math.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace rglru {

namespace {

constexpr int kHalo = 3;
constexpr int kXRows = kScanTC + kHalo;

template <typename T> struct SV;
template <> struct SV<__nv_bfloat16> {
  static constexpr int V = 4;
  static constexpr bool kAccurate = false;
};
template <> struct SV<float> {
  static constexpr int V = 2;
  static constexpr bool kAccurate = true;
};

constexpr int kGroups = 32;                           // channel groups: the lanes of a compute warp
constexpr int kSub = kScanSub;                        // sub-chunks: one compute warp each
constexpr int kL = kScanTC / kSub;                    // steps per sub-chunk
constexpr int kComputeWarps = kSub;                   // 16
constexpr int kComputeThreads = kGroups * kSub;       // 512
// The coefficient scan splits its compute warps into two groups of 8 that take alternate
// tiles; a warp then folds and replays 8 steps, so a tile has 8 sub-chunk maps, not 16.
constexpr int kLC = 8;                                // steps per coefficient sub-chunk
constexpr int kSubC = kScanTC / kLC;                  // 8 sub-chunks: one warp of the group each
static_assert(2 * kSubC == kComputeWarps, "two compute groups");
// Look-back groups of two warps: the coefficient scan's tiles are short, so two groups take
// alternate tiles (tile k goes to group k mod 2) and one tile's look-back overlaps the next
// one's. (Its 21 warps put 6 on some scheduler partition, which leaves a thread 80
// registers; 19 warps leave 96.)
template <bool kCoef> constexpr int look_groups() { return kCoef ? 2 : 1; }
template <bool kCoef> constexpr int look_threads() { return 64; }  // per group
template <bool kCoef> constexpr int threads_of() {
  return kComputeThreads + look_groups<kCoef>() * look_threads<kCoef>() + 32;  // + one producer warp
}
// named barriers (id 0 is __syncthreads, which the roles never use after the prologue):
// kBarMaps + (tile k mod 2, or mod 4 for two compute groups); compute warps arrive once
// phase 1 is done, look-back warps wait
constexpr int kBarMaps = 1;

// kCoef: the stage holds only the two coefficient blocks (d = 1 − a_t fp16, b_t bf16), which
// need neither x nor parameters, so the ring is deeper.
template <typename T, bool kGate, bool kCoef = false> struct SmemLayout {
  static constexpr int CW = kGroups * SV<T>::V;
  static constexpr int kStages = kCoef ? 6 : 3;
  static constexpr int kSubs = kCoef ? kSubC : kSub;   // sub-chunk maps per tile
  static constexpr int kX = kCoef ? 0 : kXRows * CW * (int)sizeof(T);
  static constexpr int kZ = kScanTC * CW * (int)sizeof(T);
  // a stage: x rows, z_a, z_x (TMA), then the tile's parameters [6][CW] f32 (taps 0..3,
  // conv bias, c·log σ(Λ)) written by the producer warp
  static constexpr int offZA = kX;
  static constexpr int offZX = kX + kZ;
  static constexpr int offPar = kX + 2 * kZ;
  static constexpr int kStage = offPar + (kCoef ? 0 : 6 * CW * 4);
  // Tile k uses map buffer, maps barrier and states barrier number k mod kMapBufs. Each is
  // in use from the tile's phase 1 until its phase 3 has read the handed-out states, and a
  // role reaches the next tile with the same number only after that: with one compute
  // group, tile k + 2 starts phase 1 after phase 3 of tile k; with two groups (each on
  // every other tile) that holds for tile k + 4, so each group needs two of each.
  static constexpr int kMapBufs = kCoef ? 4 : 2;
  static constexpr int offMaps = kStages * kStage;     // [kMapBufs][A | B][kSubs][CW] f32
  static constexpr int kMaps = 2 * kSubs * CW * 4;
  static constexpr int kBytes = offMaps + kMapBufs * kMaps;
  static constexpr int kAlloc = kBytes + 128;          // slack to align the base to 128 bytes
  static constexpr uint32_t kTxXZ = kX + 2 * kZ;
  static_assert(kX % 128 == 0 && kStage % 128 == 0, "TMA destinations 128-byte aligned");
  static_assert(kAlloc <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ void bar_sync_n(int id, int n) {  // id is warp-uniform
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void bar_arrive_n(int id, int n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* m, uint64_t* bar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u32(uint32_t* p, uint32_t v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Published carries are stored as their bit pattern XOR 0x7FFFFFFF: exact and reversible
// for every value but the NaN pattern 0x7FFFFFFF, whose image would be zero; that one is
// stored as the image of another NaN, so zeroed memory reads as "not published yet", no
// published word is zero, and every non-NaN value round-trips bit for bit.
constexpr uint32_t kCarryKey = 0x7FFFFFFFu;
__device__ __forceinline__ uint32_t enc(float v) {
  const uint32_t w = __float_as_uint(v) ^ kCarryKey;
  return w != 0u ? w : 1u;
}
__device__ __forceinline__ float dec(uint32_t w) { return __uint_as_float(w ^ kCarryKey); }

// A tile's map h ↦ A·h + B over its 64 steps (its aggregate), published as soon as its
// phase 1 is done — before its own look-back — as one 64-bit word per channel: enc(A) in the
// low half (never zero, so zeroed memory reads as "not yet"), the bits of B in the high half.
__device__ __forceinline__ uint64_t enc_agg(float A, float B) {
  return (uint64_t)enc(A) | ((uint64_t)__float_as_uint(B) << 32);
}
__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u64(uint64_t* p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
// predecessors whose words one round of the look-back reads at once
constexpr int kLookWindow = 8;

struct TileCoord {
  int chunk, b, cblk;  // chunk < 0: no tile (the end of a CTA's sequence)
  int tix;             // carry slot: ((b · n_cblk + cblk) · n_chunks + chunk) < n_tiles
};
__device__ __forceinline__ TileCoord coord_of(int ticket, const ScanArgs& a) {
  TileCoord c;
  const int per_chunk = a.B * a.n_cblk;
  c.chunk = ticket / per_chunk;
  const int rem = ticket - c.chunk * per_chunk;
  c.b = rem / a.n_cblk;
  c.cblk = rem - c.b * a.n_cblk;
  c.tix = (c.b * a.n_cblk + c.cblk) * a.n_chunks + c.chunk;
  return c;
}

template <typename T, bool kGate, bool kCoef>
__device__ __forceinline__ void issue_tile_loads(uint8_t* stage, uint64_t* bar, const ScanMaps& m, const ScanArgs& a,
                                                 const TileCoord& c) {
  using Ly = SmemLayout<T, kGate, kCoef>;
  constexpr int CW = Ly::CW;
  mbar_arrive_expect_tx(bar, Ly::kTxXZ);
  const int c0 = c.cblk * CW;
  const int t0 = c.chunk * kScanTC;
  if constexpr (!kCoef) tma_load_3d(stage, &m.x, bar, c0, t0 - kHalo, c.b);
  const int zcol = (c0 / kGateBlock) * 2 * kGateBlock + (c0 % kGateBlock);
  const int zrow = c.b * a.T + t0;
  tma_load_2d(stage + Ly::offZA, &m.z, bar, zcol, zrow);
  tma_load_2d(stage + Ly::offZX, &m.z, bar, zcol + kGateBlock, zrow);
}

// V consecutive elements as floats, and back (shared or global memory).
__device__ __forceinline__ void ldv(const __nv_bfloat16* p, float (&f)[4]) {
  const uint2 r = *reinterpret_cast<const uint2*>(p);
  f[0] = bf16lo(r.x); f[1] = bf16hi(r.x); f[2] = bf16lo(r.y); f[3] = bf16hi(r.y);
}
__device__ __forceinline__ void ldv(const float* p, float (&f)[2]) {
  const float2 r = *reinterpret_cast<const float2*>(p);
  f[0] = r.x; f[1] = r.y;
}
__device__ __forceinline__ void stv(__nv_bfloat16* p, const float (&f)[4]) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]));
}
__device__ __forceinline__ void stv(float* p, const float (&f)[2]) {
  *reinterpret_cast<float2*>(p) = make_float2(f[0], f[1]);
}
// read-only global loads of an input row segment
__device__ __forceinline__ void ldv_nc(const __nv_bfloat16* p, float (&f)[4]) {
  const uint2 r = __ldg(reinterpret_cast<const uint2*>(p));
  f[0] = bf16lo(r.x); f[1] = bf16hi(r.x); f[2] = bf16lo(r.y); f[3] = bf16hi(r.y);
}
__device__ __forceinline__ void ldv_nc(const float* p, float (&f)[2]) {
  const float2 r = __ldg(reinterpret_cast<const float2*>(p));
  f[0] = r.x; f[1] = r.y;
}
// streaming store of an output row segment (y is not re-read by this kernel)
__device__ __forceinline__ void stv_cs(__nv_bfloat16* p, const float (&f)[4]) {
  __stcs(reinterpret_cast<uint2*>(p), make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3])));
}
__device__ __forceinline__ void stv_cs(float* p, const float (&f)[2]) {
  __stcs(reinterpret_cast<float2*>(p), make_float2(f[0], f[1]));
}
// V float32 values from shared memory
template <int V> __device__ __forceinline__ void ldf(const float* p, float (&f)[V]);
template <> __device__ __forceinline__ void ldf<4>(const float* p, float (&f)[4]) {
  const float4 r = *reinterpret_cast<const float4*>(p);
  f[0] = r.x; f[1] = r.y; f[2] = r.z; f[3] = r.w;
}
template <> __device__ __forceinline__ void ldf<2>(const float* p, float (&f)[2]) {
  const float2 r = *reinterpret_cast<const float2*>(p);
  f[0] = r.x; f[1] = r.y;
}
template <int V> __device__ __forceinline__ void stf(float* p, const float (&f)[V]);
template <> __device__ __forceinline__ void stf<4>(float* p, const float (&f)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
}
template <> __device__ __forceinline__ void stf<2>(float* p, const float (&f)[2]) {
  *reinterpret_cast<float2*>(p) = make_float2(f[0], f[1]);
}

// −expm1(x) for x ∈ [−1/8, 0] on a pair of lanes: the Taylor series of e^x − 1 about 0
// to degree 6, −x (1 + x/2 + x²/6 + x³/24 + x⁴/120 + x⁵/720); the first omitted term is
// below 5e-8 of the result on this interval.
__device__ __forceinline__ float2 neg_expm1_eighth2(float2 x) {
  float2 p = __ffma2_rn(x, make_float2(1.0f / 720.0f, 1.0f / 720.0f), make_float2(1.0f / 120.0f, 1.0f / 120.0f));
  p = __ffma2_rn(p, x, make_float2(1.0f / 24.0f, 1.0f / 24.0f));
  p = __ffma2_rn(p, x, make_float2(1.0f / 6.0f, 1.0f / 6.0f));
  p = __ffma2_rn(p, x, make_float2(0.5f, 0.5f));
  p = __ffma2_rn(p, x, make_float2(1.0f, 1.0f));
  return __fmul2_rn(make_float2(-x.x, -x.y), p);
}

// Fast gate math for two channels: d = 1 − a_t and b_t = √(1−a_t²)·i·u.
// r = σ(z_a) (ex2 + rcp); log a_t = r·cla; d = −expm1(log a_t) (polynomial on [−1/8, 0],
// 1 − ex2 beyond); 1 − a_t² = d (2 − d); √(1−a_t²)·i = q·rsqrt(q (1 + e^{−z_x})² + 1e-30)
// (the tiny term keeps q = 0 exact: 0·finite). Four MUFU operations per element.
template <bool kSmall = false>
__device__ __forceinline__ void gate_fast2(float2 za, float2 zx, float2 cla, float2 u, float2& d, float2& bt) {
  const float2 na = __fmul2_rn(za, make_float2(-kLog2e, -kLog2e));
  const float2 nx = __fmul2_rn(zx, make_float2(-kLog2e, -kLog2e));
  const float2 ea = __fadd2_rn(make_float2(ex2_approx(na.x), ex2_approx(na.y)), make_float2(1.0f, 1.0f));
  const float2 r = make_float2(rcp_approx(ea.x), rcp_approx(ea.y));
  const float2 la = __fmul2_rn(r, cla);
  if (kSmall || fminf(la.x, la.y) >= -0.125f) {
    // kSmall: the caller knows c·log σ(Λ) ≥ −1/8, hence log a_t = r·c·log σ(Λ) ≥ −1/8
    d = neg_expm1_eighth2(la);
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

// A producer lane's share of one tile's parameters: PV = CW / 32 consecutive channels.
template <int PV> struct ParRegs {
  float w[4][PV], cb[PV], lam[PV];
};
// Issues the loads for channels c .. c+PV-1 (taps 0..3, conv bias, Λ); channels past R
// read as 0 (c is a multiple of PV and R of 8, so a lane's channels are all in or all out).
// Nothing here waits for the values.
template <int PV>
__device__ __forceinline__ void load_params(ParRegs<PV>& p, int c, const ScanArgs& a) {
#pragma unroll
  for (int v = 0; v < PV; ++v) {
    p.w[0][v] = p.w[1][v] = p.w[2][v] = p.w[3][v] = 0.0f;
    p.cb[v] = p.lam[v] = 0.0f;
  }
  if (c < a.R) {
    const int R = a.R;
#pragma unroll
    for (int v = 0; v < PV; ++v) {
#pragma unroll
      for (int i = 0; i < 4; ++i) p.w[i][v] = __ldg(a.conv_w + i * R + c + v);
      p.cb[v] = __ldg(a.conv_b + c + v);
      p.lam[v] = __ldg(a.Lambda + c + v);
    }
  }
}
// Writes them into a stage's parameter block [6][CW] at channel slot jj, with Λ turned into
// c·log σ(Λ) (0 for channels past R, which makes their steps identities).
template <int PV>
__device__ __forceinline__ void store_params(float* sPar, int CW, int jj, bool in_range, const ParRegs<PV>& p) {
  float cla[PV];
#pragma unroll
  for (int v = 0; v < PV; ++v) cla[v] = in_range ? decay_log_coeff(p.lam[v]) : 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) stf<PV>(sPar + i * CW + jj, p.w[i]);
  stf<PV>(sPar + 4 * CW + jj, p.cb);
  stf<PV>(sPar + 5 * CW + jj, cla);
}

// Phase 1 of one tile for compute thread (g, s): conv, gates, log-space decay and the fold
// of the sub-chunk's 4 steps into (A, B); the replay values go over the z_a, z_x slots the
// thread read them from (no other thread reads those slots).
// kFast: every step of the sub-chunk is inside [0, T) and every channel of the warp has
// c·log σ(Λ) ≥ −1/8, so neither the identity-step mask nor the wide decay path is needed.
template <typename T, bool kGate, bool kFast>
__device__ __forceinline__ void phase1_body(uint8_t* stage, float* mA, float* mB, const TileCoord& tc, int g, int s,
                                            const ScanArgs& a) {
  using Ly = SmemLayout<T, kGate>;
  constexpr int V = SV<T>::V;
  constexpr int CW = Ly::CW;
  constexpr bool kAcc = SV<T>::kAccurate;
  const T* sx = reinterpret_cast<const T*>(stage);
  T* sza = reinterpret_cast<T*>(stage + Ly::offZA);
  T* szx = reinterpret_cast<T*>(stage + Ly::offZX);
  const float* sP = reinterpret_cast<const float*>(stage + Ly::offPar);
  const int cc = g * V;
  const int c0 = tc.cblk * CW + cc;
  const int t_start = tc.chunk * kScanTC + s * kL;

  float W0[V], W1[V], W2[V], W3[V], CB[V], CL[V];
  ldf<V>(sP + 0 * CW + cc, W0);
  ldf<V>(sP + 1 * CW + cc, W1);
  ldf<V>(sP + 2 * CW + cc, W2);
  ldf<V>(sP + 3 * CW + cc, W3);
  ldf<V>(sP + 4 * CW + cc, CB);
  ldf<V>(sP + 5 * CW + cc, CL);
  float xm3[V], xm2[V], xm1[V];
  if (tc.chunk == 0 && s == 0 && a.state0 != nullptr) {
    // conv history of the first steps: the caller's state, oldest row first
#pragma unroll
    for (int v = 0; v < V; ++v) xm3[v] = xm2[v] = xm1[v] = 0.0f;
    if (c0 < a.R) {
      const T* st = static_cast<const T*>(a.state0) + (int64_t)tc.b * 3 * a.R + c0;
      ldv(st, xm3);
      ldv(st + a.R, xm2);
      ldv(st + 2 * a.R, xm1);
    }
  } else {
    ldv(sx + (s * kL + 0) * CW + cc, xm3);
    ldv(sx + (s * kL + 1) * CW + cc, xm2);
    ldv(sx + (s * kL + 2) * CW + cc, xm1);
  }
  float A[V], B[V];
#pragma unroll
  for (int v = 0; v < V; ++v) { A[v] = 1.0f; B[v] = 0.0f; }
#pragma unroll
  for (int l = 0; l < kL; ++l) {
    const int row = s * kL + l;
    float xc[V], za[V], zx[V];
    ldv(sx + (row + kHalo) * CW + cc, xc);
    ldv(sza + row * CW + cc, za);
    ldv(szx + row * CW + cc, zx);
    const bool tv = kFast || (t_start + l) < a.T;
    float u[V];
#pragma unroll
    for (int v = 0; v < V; v += 2) {
      float2 uu = __ffma2_rn(make_float2(W0[v], W0[v + 1]), make_float2(xm3[v], xm3[v + 1]), make_float2(CB[v], CB[v + 1]));
      uu = __ffma2_rn(make_float2(W1[v], W1[v + 1]), make_float2(xm2[v], xm2[v + 1]), uu);
      uu = __ffma2_rn(make_float2(W2[v], W2[v + 1]), make_float2(xm1[v], xm1[v + 1]), uu);
      uu = __ffma2_rn(make_float2(W3[v], W3[v + 1]), make_float2(xc[v], xc[v + 1]), uu);
      u[v] = uu.x;
      u[v + 1] = uu.y;
    }
    float at[V], r0[V], bt[V];  // r0: what goes over z_a (a_t, or 1 − a_t on the bf16 path)
    if constexpr (kAcc) {
#pragma unroll
      for (int v = 0; v < V; ++v) gate_accurate(za[v], zx[v], CL[v], u[v], at[v], bt[v]);
      if (!tv) {
        // steps past T are identity steps
#pragma unroll
        for (int v = 0; v < V; ++v) { at[v] = 1.0f; bt[v] = 0.0f; }
      }
#pragma unroll
      for (int v = 0; v < V; ++v) r0[v] = at[v];
    } else {
      if (!tv) {
        // steps past T: r = σ(−∞) = 0 makes a_t = 1 and b_t = 0 (identity steps)
#pragma unroll
        for (int v = 0; v < V; ++v) za[v] = -INFINITY;
      }
#pragma unroll
      for (int v = 0; v < V; v += 2) {
        float2 d, b2;
        gate_fast2<kFast>(make_float2(za[v], za[v + 1]), make_float2(zx[v], zx[v + 1]),
                          make_float2(CL[v], CL[v + 1]), make_float2(u[v], u[v + 1]), d, b2);
        r0[v] = d.x;
        r0[v + 1] = d.y;
        bt[v] = b2.x;
        bt[v + 1] = b2.y;
        at[v] = 1.0f - d.x;
        at[v + 1] = 1.0f - d.y;
      }
    }
    stv(sza + row * CW + cc, r0);
    stv(szx + row * CW + cc, bt);
    // fold: (A, B) ← (a·A, a·B + b)
#pragma unroll
    for (int v = 0; v < V; v += 2) {
      const float2 a2 = make_float2(at[v], at[v + 1]);
      const float2 nb = __ffma2_rn(a2, make_float2(B[v], B[v + 1]), make_float2(bt[v], bt[v + 1]));
      const float2 na = __fmul2_rn(a2, make_float2(A[v], A[v + 1]));
      A[v] = na.x; A[v + 1] = na.y;
      B[v] = nb.x; B[v + 1] = nb.y;
    }
#pragma unroll
    for (int v = 0; v < V; ++v) {
      xm3[v] = xm2[v];
      xm2[v] = xm1[v];
      xm1[v] = xc[v];
    }
  }
  stf<V>(mA + s * CW + cc, A);
  stf<V>(mB + s * CW + cc, B);
}

// The coefficients of one sub-chunk as one compute thread holds them: kLC steps × 4
// channels of d (packed fp16 pairs) and of b (packed bf16 pairs); bf16 IO only.
struct CoefRegs {
  uint32_t d[kLC][2], b[kLC][2];
};

// Reads the thread's coefficients of the tile out of the stage (after which the stage may
// be refilled).
template <bool kGate>
__device__ __forceinline__ void coef_load(const uint8_t* stage, int g, int s, CoefRegs& r) {
  using Ly = SmemLayout<__nv_bfloat16, kGate, true>;
  constexpr int CW = Ly::CW;
  const __half* sd = reinterpret_cast<const __half*>(stage + Ly::offZA);
  const __half* sb = reinterpret_cast<const __half*>(stage + Ly::offZX);
  const int cc = g * 4;
#pragma unroll
  for (int l = 0; l < kLC; ++l) {
    const int row = s * kLC + l;
    const uint2 vd = *reinterpret_cast<const uint2*>(sd + row * CW + cc);
    const uint2 vb = *reinterpret_cast<const uint2*>(sb + row * CW + cc);
    r.d[l][0] = vd.x; r.d[l][1] = vd.y;
    r.b[l][0] = vb.x; r.b[l][1] = vb.y;
  }
}
__device__ __forceinline__ float2 h2f(uint32_t w) {
  return __half22float2(*reinterpret_cast<const __half2*>(&w));
}
// a packed bf16 pair as two floats (the low half is the first element)
__device__ __forceinline__ float2 bf2f(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// Phase 1 of the coefficient scan from registers: fold the sub-chunk's 4 steps,
// (A, B) ← (a·A, a·B + b) with a = 1 − d, into its map. Steps past T are identity steps.
template <bool kGate>
__device__ __forceinline__ void coef_fold(const CoefRegs& r, float* mA, float* mB, const TileCoord& tc, int g, int s,
                                          const ScanArgs& a) {
  constexpr int CW = SmemLayout<__nv_bfloat16, kGate, true>::CW;
  const int cc = g * 4;
  const int t_start = tc.chunk * kScanTC + s * kLC;
  float2 A[2] = {make_float2(1.0f, 1.0f), make_float2(1.0f, 1.0f)};
  float2 B[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
  const bool whole = t_start + kLC <= a.T;
#pragma unroll
  for (int l = 0; l < kLC; ++l) {
    if (whole || t_start + l < a.T) {
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        const float2 d2 = h2f(r.d[l][p]);
        const float2 a2 = make_float2(1.0f - d2.x, 1.0f - d2.y);
        B[p] = __ffma2_rn(a2, B[p], bf2f(r.b[l][p]));
        A[p] = __fmul2_rn(a2, A[p]);
      }
    }
  }
  *reinterpret_cast<float4*>(mA + s * CW + cc) = make_float4(A[0].x, A[0].y, A[1].x, A[1].y);
  *reinterpret_cast<float4*>(mB + s * CW + cc) = make_float4(B[0].x, B[0].y, B[1].x, B[1].y);
}

// Phase 3 of the coefficient scan: replay the sub-chunk from its incoming state (mH) with
// the coefficients read again from the stage, and write y (times GeLU of the gate branch
// for the gated scan). The 8 steps go in two halves, each with its coefficient and gate
// loads issued before its arithmetic, so that at most half of them are held at a time.
template <bool kGate>
__device__ __forceinline__ void coef_replay(const uint8_t* stage, const float* mH, const TileCoord& tc, int g, int s,
                                            const ScanArgs& a) {
  using Ly = SmemLayout<__nv_bfloat16, kGate, true>;
  constexpr int CW = Ly::CW;
  constexpr int kHalf = kLC / 2;
  const __half* sd = reinterpret_cast<const __half*>(stage + Ly::offZA);
  const __half* sb = reinterpret_cast<const __half*>(stage + Ly::offZX);
  const int cc = g * 4;
  const int c0 = tc.cblk * CW + cc;
  const int t_start = tc.chunk * kScanTC + s * kLC;
  const float4 h4 = *reinterpret_cast<const float4*>(mH + s * CW + cc);
  float2 h[2] = {make_float2(h4.x, h4.y), make_float2(h4.z, h4.w)};
  __nv_bfloat16* __restrict__ y = static_cast<__nv_bfloat16*>(a.y);
  const bool in_range = c0 < a.R;
#pragma unroll
  for (int l0 = 0; l0 < kLC; l0 += kHalf) {
    uint32_t d[kHalf][2], b[kHalf][2];
    float gg[kGate ? kHalf : 1][4];
#pragma unroll
    for (int l = 0; l < kHalf; ++l) {
      const int row = s * kLC + l0 + l;
      const uint2 vd = *reinterpret_cast<const uint2*>(sd + row * CW + cc);
      const uint2 vb = *reinterpret_cast<const uint2*>(sb + row * CW + cc);
      d[l][0] = vd.x; d[l][1] = vd.y;
      b[l][0] = vb.x; b[l][1] = vb.y;
      if constexpr (kGate) {
#pragma unroll
        for (int v = 0; v < 4; ++v) gg[l][v] = 0.0f;
        const int t = t_start + l0 + l;
        if (in_range && t < a.T)
          ldv_nc(static_cast<const __nv_bfloat16*>(a.g) + ((int64_t)tc.b * a.T + t) * a.R + c0, gg[l]);
      }
    }
#pragma unroll
    for (int l = 0; l < kHalf; ++l) {
      float o[4];
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        const float2 d2 = h2f(d[l][p]);
        const float2 a2 = make_float2(1.0f - d2.x, 1.0f - d2.y);
        h[p] = __ffma2_rn(a2, h[p], bf2f(b[l][p]));
        o[2 * p] = h[p].x;
        o[2 * p + 1] = h[p].y;
      }
      if constexpr (kGate) {
#pragma unroll
        for (int v = 0; v < 4; ++v) o[v] *= gelu_exact(gg[l][v]);
      }
      const int t = t_start + l0 + l;
      if (in_range && t < a.T) stv_cs(y + ((int64_t)tc.b * a.T + t) * a.R + c0, o);
    }
  }
}

template <typename T, bool kGate>
__device__ __forceinline__ void phase1(uint8_t* stage, float* mA, float* mB, const TileCoord& tc, int g, int s,
                                       const ScanArgs& a) {
  using Ly = SmemLayout<T, kGate>;
  constexpr int V = SV<T>::V;
  bool fast = false;
  if constexpr (!SV<T>::kAccurate) {
    const float* CL = reinterpret_cast<const float*>(stage + Ly::offPar) + 5 * Ly::CW + g * V;
    bool small = true;
#pragma unroll
    for (int v = 0; v < V; ++v) small = small && CL[v] >= -0.125f;
    fast = __all_sync(0xffffffffu, small) && tc.chunk * kScanTC + (s + 1) * kL <= a.T;
  }
  if (fast)
    phase1_body<T, kGate, true>(stage, mA, mB, tc, g, s, a);
  else
    phase1_body<T, kGate, false>(stage, mA, mB, tc, g, s, a);
}

// Phase 3 of one tile for compute thread (g, s): replay the sub-chunk from its incoming
// state (mH) and write y (times GeLU of the gate branch for the gated scan). Every
// shared-memory read comes first and is followed by the proxy fence that lets the stage be
// refilled by asynchronous copies; only then are the global stores issued, so the fence
// never waits for them.
template <typename T, bool kGate>
__device__ __forceinline__ void phase3(const uint8_t* stage, const float* mH, const TileCoord& tc, int g, int s,
                                       const ScanArgs& a) {
  using Ly = SmemLayout<T, kGate>;
  constexpr int V = SV<T>::V;
  constexpr int CW = Ly::CW;
  constexpr bool kAcc = SV<T>::kAccurate;
  const T* sza = reinterpret_cast<const T*>(stage + Ly::offZA);
  const T* szx = reinterpret_cast<const T*>(stage + Ly::offZX);
  const int cc = g * V;
  const int c0 = tc.cblk * CW + cc;
  const int t_start = tc.chunk * kScanTC + s * kL;
  float h[V];
  float r0[kL][V], bt[kL][V], gg[kGate ? kL : 1][V];
  if constexpr (kGate) {
    // the gate branch comes straight from global memory; its loads are issued first
    const T* gsrc = static_cast<const T*>(a.g);
#pragma unroll
    for (int l = 0; l < kL; ++l) {
#pragma unroll
      for (int v = 0; v < V; ++v) gg[l][v] = 0.0f;
      if (c0 < a.R && t_start + l < a.T) ldv_nc(gsrc + ((int64_t)tc.b * a.T + t_start + l) * a.R + c0, gg[l]);
    }
  }
  ldf<V>(mH + s * CW + cc, h);
#pragma unroll
  for (int l = 0; l < kL; ++l) {
    const int row = s * kL + l;
    ldv(sza + row * CW + cc, r0[l]);
    ldv(szx + row * CW + cc, bt[l]);
  }
  fence_proxy_async_smem();
  if (c0 >= a.R) return;
  T* __restrict__ y = static_cast<T*>(a.y);
#pragma unroll
  for (int l = 0; l < kL; ++l) {
    float o[V];
#pragma unroll
    for (int v = 0; v < V; v += 2) {
      const float2 a2 =
          kAcc ? make_float2(r0[l][v], r0[l][v + 1]) : make_float2(1.0f - r0[l][v], 1.0f - r0[l][v + 1]);
      const float2 h2 = __ffma2_rn(a2, make_float2(h[v], h[v + 1]), make_float2(bt[l][v], bt[l][v + 1]));
      h[v] = o[v] = h2.x;
      h[v + 1] = o[v + 1] = h2.y;
    }
    if constexpr (kGate) {
#pragma unroll
      for (int v = 0; v < V; ++v) o[v] *= gelu_exact(gg[l][v]);
    }
    const int t = t_start + l;
    if (t < a.T) stv_cs(y + ((int64_t)tc.b * a.T + t) * a.R + c0, o);
  }
}

// Look-back, first half, for thread j's NCH channel slots j, j + CW/NCH, ...: the state
// entering the tile is the inclusive state its predecessor (the previous time chunk of the
// same batch row and channel block) publishes, or h0 for the first chunk. It needs nothing
// of this tile, so its first read is issued before phase 1 of the tile is done and is only
// waited for (lookback_end) once the tile's maps are composed. Channels past R (the padding
// of the last channel block) neither wait for nor publish a state, so whatever their
// padding inputs hold cannot stall a tile.
template <typename T, bool kGate, int NCH>
__device__ __forceinline__ void lookback_begin(const TileCoord& tc, int j, const ScanArgs& a, uint32_t (&w)[NCH],
                                               float (&hin)[NCH]) {
  constexpr int CW = SmemLayout<T, kGate>::CW;
  constexpr int kStride = CW / NCH;
  if (tc.chunk == 0) {
#pragma unroll
    for (int n = 0; n < NCH; ++n) {
      const int c = tc.cblk * CW + j + n * kStride;
      hin[n] = (a.h0 != nullptr && c < a.R) ? a.h0[(int64_t)tc.b * a.R + c] : 0.0f;
      w[n] = 1u;
    }
    return;
  }
  // the read is unconditional (every channel slot of a tile exists), so nothing waits for
  // its result before lookback_end
  const uint32_t* src = a.carry_incl + (int64_t)(tc.tix - 1) * CW + j;
#pragma unroll
  for (int n = 0; n < NCH; ++n) w[n] = ld_relaxed_u32(src + n * kStride);
}
// Decoupled look-back. The state entering tile k is the inclusive state of its predecessor
// chunk k − 1. If that is not published yet, the walk goes back over the predecessors whose
// aggregates (A, B) are (kLookWindow of them per round trip) to the nearest published
// inclusive state h_m, then replays forward: h ← fmaf(A_j, h, B_j) for j = m + 1 … k − 1 —
// the very operation by which tile j forms its own inclusive state from its incoming one,
// on the same bits. So the state a tile starts from does not depend on which words had been
// published when it looked (the result is deterministic, whatever the timing), while no tile
// waits for more than the aggregates of its predecessors. Chunk 0 publishes its inclusive
// state straight away, so every walk ends; a round that finds neither word of the next
// predecessor reads it again, within the deadline.
template <typename T, bool kGate, int NCH>
__device__ __forceinline__ void lookback_end(const TileCoord& tc, int j, const ScanArgs& a, uint32_t (&w)[NCH],
                                             float (&hin)[NCH]) {
  constexpr int CW = SmemLayout<T, kGate>::CW;
  constexpr int kStride = CW / NCH;
  if (tc.chunk == 0) return;
  int depth[NCH];  // > 0: searching (the predecessor depth chunks back is next); ≤ 0: found
  int rest[NCH];   // once found: the predecessors still to replay are depths rest − 1 … 1
  bool all = true;
#pragma unroll
  for (int n = 0; n < NCH; ++n) {
    const bool pad = tc.cblk * CW + j + n * kStride >= a.R;  // no state: neither waits nor publishes
    depth[n] = pad ? 0 : (w[n] != 0u ? -1 : 1);
    rest[n] = 1;
    hin[n] = pad ? 0.0f : (w[n] != 0u ? dec(w[n]) : 0.0f);
    all = all && depth[n] <= 0;
  }
  if (all) return;
  // 1. the nearest published inclusive state, for every channel still searching
  const long long t0 = clock64();
  bool timed_out = false;
  while (true) {
    all = true;
#pragma unroll
    for (int n = 0; n < NCH; ++n) {
      if (depth[n] <= 0) continue;
      const int left = tc.chunk - depth[n] + 1;  // predecessors at this depth or older: chunks 0 … left − 1
      const int64_t slot0 = (int64_t)(tc.tix - depth[n]) * CW + j + n * kStride;
      uint32_t wi[kLookWindow];
      uint64_t ga[kLookWindow];
#pragma unroll
      for (int i = 0; i < kLookWindow; ++i) {
        wi[i] = i < left ? ld_relaxed_u32(a.carry_incl + slot0 - (int64_t)i * CW) : 0u;
        ga[i] = i < left ? ld_relaxed_u64(a.carry_agg + slot0 - (int64_t)i * CW) : 0ull;
      }
      const int d_start = depth[n];
      int found = -1;
#pragma unroll
      for (int i = 0; i < kLookWindow; ++i) {
        if (found < 0 && wi[i] != 0u) found = i;
        if (found < 0 && ga[i] == 0ull) break;
        if (found < 0) ++depth[n];
      }
      if (found >= 0) {
        // the inclusive state found, then the window's aggregates in front of it, oldest first
        uint32_t wf = 0u;
#pragma unroll
        for (int i = 0; i < kLookWindow; ++i)
          if (i == found) wf = wi[i];
        float h = dec(wf);
#pragma unroll
        for (int i = kLookWindow - 1; i >= 0; --i)
          if (i < found) h = fmaf(dec((uint32_t)ga[i]), h, __uint_as_float((uint32_t)(ga[i] >> 32)));
        hin[n] = h;
        rest[n] = d_start;
        depth[n] = -1;
      }
      all = all && depth[n] <= 0;
    }
    if (all) break;
    if (clock64() - t0 > kWaitCycles) {
      atomicOr(a.status, kStatusTimeout);
      timed_out = true;
      break;
    }
  }
  // 2. replay the predecessors of the earlier windows (depths rest − 1 … 1), oldest first
#pragma unroll
  for (int n = 0; n < NCH; ++n) {
    if (timed_out && depth[n] > 0) continue;
    const int64_t ch = j + n * kStride;
    for (int d0 = rest[n] - 1; d0 >= 1; d0 -= kLookWindow) {
      uint64_t ga[kLookWindow];
#pragma unroll
      for (int i = 0; i < kLookWindow; ++i)
        ga[i] = d0 - i >= 1 ? ld_relaxed_u64(a.carry_agg + (int64_t)(tc.tix - (d0 - i)) * CW + ch) : 0ull;
#pragma unroll
      for (int i = 0; i < kLookWindow; ++i)
        if (d0 - i >= 1)
          hin[n] = fmaf(dec((uint32_t)ga[i]), hin[n], __uint_as_float((uint32_t)(ga[i] >> 32)));
    }
  }
}

// Look-back, second half, once phase 1 of the tile is done: composes the S sub-chunk maps
// (mA, mB) into the tile's map, waits for the incoming state, publishes the tile's inclusive
// state A·h_in + B at once (the next chunk waits for it), writes h_T for the last chunk, and
// then leaves each sub-chunk's incoming state in mB. mA and mB are separate buffers and each
// slot is read before it is overwritten, so the reads of the second pass need not wait for
// its stores.
template <typename T, bool kGate, int NCH, int S>
__device__ __forceinline__ void lookback_finish(const float* __restrict__ mA, float* __restrict__ mB,
                                                const TileCoord& tc, int j, const ScanArgs& a, uint32_t (&w)[NCH],
                                                float (&hin)[NCH]) {
  constexpr int CW = SmemLayout<T, kGate>::CW;
  constexpr int kStride = CW / NCH;
  const bool publish = tc.tix != a.stall_tile;
  float A[NCH], Bv[NCH];
#pragma unroll
  for (int n = 0; n < NCH; ++n) { A[n] = 1.0f; Bv[n] = 0.0f; }
#pragma unroll 8
  for (int q = 0; q < S; ++q) {
#pragma unroll
    for (int n = 0; n < NCH; ++n) {
      const float pa = mA[q * CW + j + n * kStride], pb = mB[q * CW + j + n * kStride];
      Bv[n] = fmaf(pa, Bv[n], pb);
      A[n] *= pa;
    }
  }
  // the tile's aggregate goes out before its own look-back (chunk 0 needs none: its
  // inclusive state follows at once)
  if (publish && tc.chunk > 0) {
#pragma unroll
    for (int n = 0; n < NCH; ++n) {
      const int jj = j + n * kStride;
      if (tc.cblk * CW + jj < a.R) st_relaxed_u64(a.carry_agg + (int64_t)tc.tix * CW + jj, enc_agg(A[n], Bv[n]));
    }
  }
  lookback_end<T, kGate, NCH>(tc, j, a, w, hin);
#pragma unroll
  for (int n = 0; n < NCH; ++n) {
    const int jj = j + n * kStride;
    const int c = tc.cblk * CW + jj;
    const float hout = fmaf(A[n], hin[n], Bv[n]);
    if (publish && c < a.R) st_relaxed_u32(a.carry_incl + (int64_t)tc.tix * CW + jj, enc(hout));
    if (tc.chunk == a.n_chunks - 1 && a.hT != nullptr && c < a.R) a.hT[(int64_t)tc.b * a.R + c] = hout;
  }
  // the state entering each sub-chunk
  float h[NCH];
#pragma unroll
  for (int n = 0; n < NCH; ++n) h[n] = hin[n];
#pragma unroll 8
  for (int q = 0; q < S; ++q) {
#pragma unroll
    for (int n = 0; n < NCH; ++n) {
      const int o = q * CW + j + n * kStride;
      const float pa = mA[o], pb = mB[o];
      mB[o] = h[n];
      h[n] = fmaf(pa, h[n], pb);
    }
  }
}

template <typename T, bool kGate, bool kCoef>
__global__ void __launch_bounds__(threads_of<kCoef>(), 1)
    rglru_scan_kernel(const __grid_constant__ ScanMaps maps, const ScanArgs a) {
  using Ly = SmemLayout<T, kGate, kCoef>;
  constexpr int kStages = Ly::kStages;
  // a stage is free once every compute warp is done with it — and, for the coefficient
  // scan, whose compute warps let go of a stage right after phase 1, once both look-back
  // warps have read its tile index
  constexpr int kGroups = look_groups<kCoef>();
  constexpr int kLookThreads = look_threads<kCoef>();
  constexpr int kSubs = Ly::kSubs;  // sub-chunk maps per tile
  // each tile is folded and replayed by all 16 compute warps, or for the coefficient scan
  // by one group of 8 (tile k by group k mod 2)
  constexpr int kTileWarps = kCoef ? kSubC : kComputeWarps;
  constexpr int kEmptyArrivals = kTileWarps;
  constexpr int kMapsBar = kTileWarps * 32 + kLookThreads;  // maps barrier participants
  constexpr int CW = Ly::CW;
  constexpr int PV = CW / 32;  // channels per producer lane
  constexpr int NCH = CW / kLookThreads;  // channels per look-back thread
  static_assert(CW % kLookThreads == 0 && CW % 32 == 0, "thread roles");

  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  __shared__ __align__(8) uint64_t full[kStages];   // TMA bytes + the producer's parameters
  __shared__ __align__(8) uint64_t empty[kStages];  // one arrival per compute warp after phase 3
  __shared__ __align__(8) uint64_t state[Ly::kMapBufs];  // tile k mod kMapBufs: incoming states ready
  __shared__ TileCoord s_tc[kStages];               // the tile in each stage (decoded once)
  float* maps_base = reinterpret_cast<float*>(smem + Ly::offMaps);
  const int tid = threadIdx.x;
  const int lane = tid & 31;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 2);
      mbar_init(&empty[i], kEmptyArrivals);
    }
    for (int i = 0; i < Ly::kMapBufs; ++i) mbar_init(&state[i], kLookThreads);
    fence_barrier_init();
  }
  __syncthreads();
  // launched as a programmatic dependent: the inputs and the zeroed workspace of the
  // kernels before are visible from here
  pdl_wait();
  pdl_launch_dependents();

  if (tid < kComputeThreads) {
    // ---- compute warps: phase 1 of tile k, then phase 3 of the group's previous tile ----
    // (all 16 warps on every tile, sub-chunk = warp; or for the coefficient scan, group
    // cg = warp / 8 on tiles cg, cg + 2, ..., sub-chunk = warp % 8)
    const int g = lane;
    const int warp = tid / 32;
    const int s = kCoef ? warp % kSubC : warp;
    const int k0 = kCoef ? warp / kSubC : 0;
    constexpr int dk = kCoef ? 2 : 1;
    for (int k = k0;; k += dk) {
      const int st = k % kStages;
      if (!mbar_wait_sleep(&full[st], (uint32_t)(k / kStages) & 1u)) {
        if (lane == 0) atomicOr(a.status, kStatusTimeout);
      }
      const TileCoord tc = s_tc[st];
      const bool valid = tc.chunk >= 0;
      if (valid) {
        float* mA = maps_base + (k % Ly::kMapBufs) * 2 * kSubs * CW;
        if constexpr (kCoef) {
          CoefRegs r;
          coef_load<kGate>(smem + st * Ly::kStage, g, s, r);
          coef_fold<kGate>(r, mA, mA + kSubs * CW, tc, g, s, a);
        } else {
          phase1<T, kGate>(smem + st * Ly::kStage, mA, mA + kSubs * CW, tc, g, s, a);
        }
        bar_arrive_n(kBarMaps + k % Ly::kMapBufs, kMapsBar);
      }
      if (k >= dk) {
        const int kp = k - dk;
        const int stp = kp % kStages;
        if (!mbar_wait_sleep(&state[kp % Ly::kMapBufs], (uint32_t)(kp / Ly::kMapBufs) & 1u)) {
          if (lane == 0) atomicOr(a.status, kStatusTimeout);
        }
        const float* mH = maps_base + (kp % Ly::kMapBufs) * 2 * kSubs * CW + kSubs * CW;
        if constexpr (kCoef) {
          // the coefficients are read again from the stage, which is released only now
          coef_replay<kGate>(smem + stp * Ly::kStage, mH, s_tc[stp], g, s, a);
        } else {
          phase3<T, kGate>(smem + stp * Ly::kStage, mH, s_tc[stp], g, s, a);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stp]);
      }
      if (!valid) break;
    }
  } else if (tid < kComputeThreads + kGroups * kLookThreads) {
    // ---- look-back warps: the incoming state of tile k is read while its phase 1 runs;
    // once phase 1 is done the tile's states are finished and published. Group gr takes
    // tiles gr, gr + kGroups, ... (the maps barrier, the maps buffer and the state barrier
    // of tile k all go by k mod 2, so each of two groups has its own) ----------------------
    const int gr = (tid - kComputeThreads) / kLookThreads;
    const int j = (tid - kComputeThreads) % kLookThreads;
    for (int k = gr;; k += kGroups) {
      const int st = k % kStages;
      if (!mbar_wait_sleep(&full[st], (uint32_t)(k / kStages) & 1u)) {
        if (j == 0) atomicOr(a.status, kStatusTimeout);
      }
      const TileCoord tc = s_tc[st];
      const bool valid = tc.chunk >= 0;
      if (!valid) break;  // the end of this CTA's tiles (the compute warps have left)
      float hin[NCH];
      uint32_t w[NCH];
      lookback_begin<T, kGate, NCH>(tc, j, a, w, hin);
      bar_sync_n(kBarMaps + k % Ly::kMapBufs, kMapsBar);
      float* mA = maps_base + (k % Ly::kMapBufs) * 2 * kSubs * CW;
      lookback_finish<T, kGate, NCH, kSubs>(mA, mA + kSubs * CW, tc, j, a, w, hin);
      mbar_arrive(&state[k % Ly::kMapBufs]);
    }
  } else {
    // ---- producer warp: tickets, TMA copies and parameters, two tiles ahead ----------
    if (lane == 0) {
      if constexpr (!kCoef) tma_prefetch_desc(&maps.x);
      tma_prefetch_desc(&maps.z);
    }
    // tickets: t_cur for the tile being loaded, t_nxt for the one after (its parameters
    // are loaded a step early), pend for the one after that (fetched a step early). A
    // CTA's first two tickets are fixed (blockIdx.x and blockIdx.x + gridDim.x, so the
    // first loads go out without a round trip to the counter); the counter hands out the
    // rest from 2·gridDim.x on. A CTA still takes its tickets in increasing order.
    const unsigned t_fixed = 2u * gridDim.x;
    unsigned pend = 0;
    if (lane == 0) pend = atomicAdd(a.ticket, 1u) + t_fixed;
    int t_cur = (int)blockIdx.x;
    int t_nxt = (int)(blockIdx.x + gridDim.x);
    ParRegs<PV> par;
    if (!kCoef && t_cur < a.n_tiles) load_params<PV>(par, coord_of(t_cur, a).cblk * CW + lane * PV, a);
    int ends = 0;
    for (int jt = 0;; ++jt) {
      const int st = jt % kStages;
      if (jt >= kStages) {
        // the stage's previous tile has been replayed by every compute warp
        if (!mbar_wait_sleep(&empty[st], (uint32_t)(jt / kStages - 1) & 1u)) {
          if (lane == 0) atomicOr(a.status, kStatusTimeout);
        }
      }
      uint8_t* stage = smem + st * Ly::kStage;
      if (lane == 0) s_tc[st] = t_cur < a.n_tiles ? coord_of(t_cur, a) : TileCoord{-1, 0, 0, 0};
      if (t_cur >= a.n_tiles) {
        // end of this CTA's tiles: release the stage with no data, once for each look-back
        // group (the compute warps stop at the first)
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&full[st]);
          mbar_arrive(&full[st]);
        }
        if (++ends == kGroups) break;
        continue;
      }
      const TileCoord tc = coord_of(t_cur, a);
      if (lane == 0) issue_tile_loads<T, kGate, kCoef>(stage, &full[st], maps, a, tc);
      if constexpr (!kCoef)
        store_params<PV>(reinterpret_cast<float*>(stage + Ly::offPar), CW, lane * PV, tc.cblk * CW + lane * PV < a.R,
                         par);
      // advance the ticket pipeline and start the next tile's parameter loads
      const int t_new = (int)__shfl_sync(0xffffffffu, pend, 0);
      if (lane == 0) pend = atomicAdd(a.ticket, 1u) + t_fixed;
      t_cur = t_nxt;
      t_nxt = t_new;
      if (!kCoef && t_cur < a.n_tiles) load_params<PV>(par, coord_of(t_cur, a).cblk * CW + lane * PV, a);
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[st]);
    }
  }
}

std::atomic<int64_t> g_stall_tile{-1};

// One CTA per SM: every CTA of the grid is resident at once, which the look-back's
// forward-progress argument needs.
template <typename T, bool kGate, bool kCoef>
cudaError_t launch_typed(const ScanArgs& a, const ScanMaps& maps, cudaStream_t s) {
  using Ly = SmemLayout<T, kGate, kCoef>;
  auto kern = rglru_scan_kernel<T, kGate, kCoef>;
  static bool ready[64] = {false};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!ready[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Ly::kAlloc);
    if (e != cudaSuccess) return e;
    int nb = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, threads_of<kCoef>(), Ly::kAlloc);
    if (e != cudaSuccess) return e;
    if (nb < 1) return cudaErrorInvalidConfiguration;
    ready[dev] = true;
  }
  const int64_t grid = std::min<int64_t>(a.n_tiles, (int64_t)num_sms());
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(threads_of<kCoef>());
  cfg.dynamicSmemBytes = Ly::kAlloc;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // the kernel waits (pdl_wait)
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, maps, a);
}

bool encode(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const cuuint64_t* dims,
            const cuuint64_t* strides, const cuuint32_t* box) {
  EncodeTiledFn fn = get_encode_tiled();
  if (fn == nullptr) return false;
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, dt, rank, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

ScanLayout scan_layout(int B, int T, int R, bool bf16) {
  ScanLayout L;
  const int cw = scan_cw(bf16);
  L.n_cblk = (R + cw - 1) / cw;
  L.n_chunks = (T + kScanTC - 1) / kScanTC;
  L.n_tiles = (int64_t)B * L.n_cblk * L.n_chunks;
  L.off_incl = 256;
  L.off_agg = L.off_incl + (((size_t)L.n_tiles * cw * 4 + 255) / 256) * 256;
  L.bytes = L.off_agg + (size_t)L.n_tiles * cw * 8;
  L.zero_bytes = L.bytes;
  return L;
}

void set_scan_stall(int64_t tile) { g_stall_tile.store(tile); }
int64_t scan_stall() { return g_stall_tile.load(); }

cudaError_t launch_scan(const ScanArgs& a_in, bool bf16, cudaStream_t s, bool coef) {
  if (coef && !bf16) return cudaErrorInvalidValue;
  ScanArgs a = a_in;
  a.stall_tile = scan_stall();
  ScanMaps maps;
  const CUtensorMapDataType dt = bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const int es = bf16 ? 2 : 4;
  const int cw = scan_cw(bf16);
  if (!coef) {
    // the coefficient scan reads no x: the gate GEMM's epilogue already formed b_t from u_t
    cuuint64_t dims[3] = {(cuuint64_t)a.R, (cuuint64_t)a.T, (cuuint64_t)a.B};
    cuuint64_t strides[2] = {(cuuint64_t)a.R * es, (cuuint64_t)a.T * a.R * es};
    cuuint32_t box[3] = {(cuuint32_t)cw, (cuuint32_t)kXRows, 1};
    if (!encode(&maps.x, dt, 3, a.x, dims, strides, box)) return cudaErrorInvalidValue;
  } else {
    memset(&maps.x, 0, sizeof(maps.x));
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)a.pitch, (cuuint64_t)a.B * a.T};
    cuuint64_t strides[1] = {(cuuint64_t)a.pitch * es};
    cuuint32_t box[2] = {(cuuint32_t)cw, (cuuint32_t)kScanTC};
    const CUtensorMapDataType zdt = coef ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : dt;  // 16-bit coefficient words
    if (!encode(&maps.z, zdt, 2, a.z, dims, strides, box)) return cudaErrorInvalidValue;
  }
  const bool gate = a.g != nullptr;
  if (coef)
    return gate ? launch_typed<__nv_bfloat16, true, true>(a, maps, s)
                : launch_typed<__nv_bfloat16, false, true>(a, maps, s);
  if (bf16)
    return gate ? launch_typed<__nv_bfloat16, true, false>(a, maps, s)
                : launch_typed<__nv_bfloat16, false, false>(a, maps, s);
  return gate ? launch_typed<float, true, false>(a, maps, s) : launch_typed<float, false, false>(a, maps, s);
}

}  // namespace rglru
