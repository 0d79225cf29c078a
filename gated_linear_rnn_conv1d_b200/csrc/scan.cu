// Fused RG-LRU scan: Conv1D recompute + σ gates + log-space decay + chunked diagonal
// recurrence; one HBM read of x and of the gate pre-activations, one write of y.
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
// and kScanTC = 64 consecutive steps. Its 256 threads are 16 channel groups (16 bytes of
// channels) × 16 sub-chunks of kScanL = 4 steps.
//
// Persistent CTAs (as many as fit on the device) take tiles in order from an atomic
// ticket — time-chunk-major, so every tile a CTA waits for was taken earlier by a running
// CTA (forward progress) — and prefetch the next ticket and the next tile's data:
//   load     one thread issues TMA bulk-tensor copies of the tile's x rows (with the
//            3-row conv halo; rows before t = 0 arrive as zeros), z_a, z_x (and g) into
//            shared memory; they land while the CTA finishes the previous tile;
//   phase 1  each thread recomputes u for its 4 steps × V channels in float32, applies
//            the gates and the log-space decay, folds the 4 steps into an affine map
//            (float32) and keeps the per-step (1 − a_t, b_t) for the replay; the x/z
//            stage is then free and the next tile's copies are issued;
//   phase 2  one thread per channel scans the 16 sub-chunk maps and gets the tile's
//            incoming state by decoupled look-back over earlier time chunks of the same
//            (b, channel block). Carries are self-validating words (an exact XOR
//            encoding whose zero is never a published value, so zeroed memory reads as
//            "not yet"), so a look-back hop is one round trip with no fence, flag or
//            barrier; waits are bounded;
//   phase 3  each thread replays its 4 steps from its incoming state and writes y.
// The per-step replay values of the bf16 path are held as bf16 pairs (1 − a_t, b_t): their
// rounding only touches y inside one 4-step run, while the carries and h_T come from the
// float32 maps.
#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cuda_bf16.h>

#include "gate_math.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace rglru {

namespace {

constexpr int kHalo = 3;
constexpr int kXRows = kScanTC + kHalo;

template <typename T> struct SV;
template <> struct SV<__nv_bfloat16> {
  static constexpr int V = 8;
  static constexpr bool kAccurate = false;
};
template <> struct SV<float> {
  static constexpr int V = 4;
  static constexpr bool kAccurate = true;
};

template <typename T, bool kGate> struct SmemLayout {
  static constexpr int CW = kScanGroups * SV<T>::V;
  static constexpr int kX = kXRows * CW * (int)sizeof(T);
  static constexpr int kZ = kScanTC * CW * (int)sizeof(T);
  static constexpr int kG = kGate ? kZ : 0;
  static constexpr int offZA = kX;
  static constexpr int offZX = offZA + kZ;
  static constexpr int offG = offZX + kZ;
  static constexpr int offA = offG + kG;
  static constexpr int offB = offA + kScanSub * CW * 4;
  static constexpr int offP = offB + kScanSub * CW * 4;   // [6][CW]: taps 0..3, conv bias, c·log σ(Λ)
  static constexpr int kBytes = offP + 6 * CW * 4;
  static constexpr int kAlloc = kBytes + 128;  // slack to align the base to 128 bytes
  static constexpr uint32_t kTxXZ = kX + 2 * kZ;
};

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
__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u32(uint32_t* p, uint32_t v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void st_relaxed_u64(uint64_t* p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Published carries are stored as their bit pattern XOR 0x7FFFFFFF: an exact, reversible
// encoding whose only zero is the image of one NaN pattern, so zeroed memory reads as
// "not published yet" and every finite value round-trips bit for bit.
constexpr uint32_t kCarryKey = 0x7FFFFFFFu;
__device__ __forceinline__ uint32_t enc(float v) { return __float_as_uint(v) ^ kCarryKey; }
__device__ __forceinline__ float dec(uint32_t w) { return __uint_as_float(w ^ kCarryKey); }

struct TileCoord {
  int chunk, b, cblk;
  int64_t tix;  // carry slot: ((b · n_cblk + cblk) · n_chunks + chunk)
};
__device__ __forceinline__ TileCoord coord_of(int ticket, const ScanArgs& a) {
  TileCoord c;
  const int per_chunk = a.B * a.n_cblk;
  c.chunk = ticket / per_chunk;
  const int rem = ticket - c.chunk * per_chunk;
  c.b = rem / a.n_cblk;
  c.cblk = rem - c.b * a.n_cblk;
  c.tix = ((int64_t)c.b * a.n_cblk + c.cblk) * a.n_chunks + c.chunk;
  return c;
}

template <typename T, bool kGate>
__device__ __forceinline__ void issue_tile_loads(uint8_t* smem, uint64_t* bar, const ScanMaps& m, const ScanArgs& a,
                                                 const TileCoord& c) {
  using Ly = SmemLayout<T, kGate>;
  constexpr int CW = Ly::CW;
  mbar_arrive_expect_tx(bar, Ly::kTxXZ + Ly::kG);
  const int c0 = c.cblk * CW;
  const int t0 = c.chunk * kScanTC;
  tma_load_3d(smem, &m.x, bar, c0, t0 - kHalo, c.b);
  const int zcol = (c0 / kGateBlock) * 2 * kGateBlock + (c0 % kGateBlock);
  const int zrow = c.b * a.T + t0;
  tma_load_2d(smem + Ly::offZA, &m.z, bar, zcol, zrow);
  tma_load_2d(smem + Ly::offZX, &m.z, bar, zcol + kGateBlock, zrow);
}

template <typename T, bool kGate>
__device__ __forceinline__ void issue_gate_load(uint8_t* smem, uint64_t* bar, const ScanMaps& m, const TileCoord& c) {
  using Ly = SmemLayout<T, kGate>;
  tma_load_3d(smem + Ly::offG, &m.g, bar, c.cblk * Ly::CW, c.chunk * kScanTC, c.b);
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
__device__ __forceinline__ void gate_fast2(float2 za, float2 zx, float2 cla, float2 u, float2& d, float2& bt) {
  const float2 na = __fmul2_rn(za, make_float2(-kLog2e, -kLog2e));
  const float2 nx = __fmul2_rn(zx, make_float2(-kLog2e, -kLog2e));
  const float2 ea = __fadd2_rn(make_float2(ex2_approx(na.x), ex2_approx(na.y)), make_float2(1.0f, 1.0f));
  const float2 r = make_float2(rcp_approx(ea.x), rcp_approx(ea.y));
  const float2 la = __fmul2_rn(r, cla);
  if (fminf(la.x, la.y) >= -0.125f) {
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

// Stages the per-channel parameters of channel block `cblk` (one thread per channel).
__device__ __forceinline__ void stage_params(float* sP, int CW, int cblk, int j, const ScanArgs& a) {
  const int c = cblk * CW + j;
  const bool ok = c < a.R;
  const int R = a.R;
  sP[0 * CW + j] = ok ? __ldg(a.conv_w + c) : 0.0f;
  sP[1 * CW + j] = ok ? __ldg(a.conv_w + R + c) : 0.0f;
  sP[2 * CW + j] = ok ? __ldg(a.conv_w + 2 * R + c) : 0.0f;
  sP[3 * CW + j] = ok ? __ldg(a.conv_w + 3 * R + c) : 0.0f;
  sP[4 * CW + j] = ok ? __ldg(a.conv_b + c) : 0.0f;
  sP[5 * CW + j] = ok ? decay_log_coeff(__ldg(a.Lambda + c)) : 0.0f;
}

// Four consecutive elements of type T from shared memory, as floats.
template <typename T> __device__ __forceinline__ float4 lds4(const T* p);
template <> __device__ __forceinline__ float4 lds4<__nv_bfloat16>(const __nv_bfloat16* p) {
  const uint2 r = *reinterpret_cast<const uint2*>(p);
  return make_float4(bf16lo(r.x), bf16hi(r.x), bf16lo(r.y), bf16hi(r.y));
}
template <> __device__ __forceinline__ float4 lds4<float>(const float* p) { return *reinterpret_cast<const float4*>(p); }

template <int V> __device__ __forceinline__ void unpack_row(const uint4& r, float (&f)[V]);
template <> __device__ __forceinline__ void unpack_row<8>(const uint4& r, float (&f)[8]) {
  f[0] = bf16lo(r.x); f[1] = bf16hi(r.x); f[2] = bf16lo(r.y); f[3] = bf16hi(r.y);
  f[4] = bf16lo(r.z); f[5] = bf16hi(r.z); f[6] = bf16lo(r.w); f[7] = bf16hi(r.w);
}
template <> __device__ __forceinline__ void unpack_row<4>(const uint4& r, float (&f)[4]) {
  f[0] = __uint_as_float(r.x); f[1] = __uint_as_float(r.y); f[2] = __uint_as_float(r.z); f[3] = __uint_as_float(r.w);
}
template <int V> __device__ __forceinline__ uint4 pack_row(const float (&f)[V]);
template <> __device__ __forceinline__ uint4 pack_row<8>(const float (&f)[8]) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
}
template <> __device__ __forceinline__ uint4 pack_row<4>(const float (&f)[4]) {
  return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
}

template <typename T, bool kGate>
__global__ void __launch_bounds__(kScanThreads, 2)
    rglru_scan_kernel(const __grid_constant__ ScanMaps maps, const ScanArgs a) {
  using Ly = SmemLayout<T, kGate>;
  constexpr int V = SV<T>::V;
  constexpr int CW = Ly::CW;
  constexpr int S = kScanSub;
  constexpr int L = kScanL;
  constexpr bool kAcc = SV<T>::kAccurate;
  static_assert(2 * CW <= kScanThreads, "phase 2 needs CW look-back threads and CW staging threads");

  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_ticket, s_next;
  float* sA = reinterpret_cast<float*>(smem + Ly::offA);
  float* sB = reinterpret_cast<float*>(smem + Ly::offB);
  float* sP = reinterpret_cast<float*>(smem + Ly::offP);
  const T* sx = reinterpret_cast<const T*>(smem);
  const T* sza = reinterpret_cast<const T*>(smem + Ly::offZA);
  const T* szx = reinterpret_cast<const T*>(smem + Ly::offZX);
  const T* sg = reinterpret_cast<const T*>(smem + Ly::offG);

  const int tid = threadIdx.x;
  const int g = tid % kScanGroups;
  const int s = tid / kScanGroups;
  const int R = a.R;
  volatile int no_abort = 0;

  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    tma_prefetch_desc(&maps.x);
    tma_prefetch_desc(&maps.z);
    if (kGate) tma_prefetch_desc(&maps.g);
    const int t = (int)atomicAdd(a.ticket, 1u);
    s_ticket = t;
    if (t < a.n_tiles) {
      const TileCoord c = coord_of(t, a);
      issue_tile_loads<T, kGate>(smem, &bar, maps, a, c);
      if (kGate) issue_gate_load<T, kGate>(smem, &bar, maps, c);
    }
    s_next = (int)atomicAdd(a.ticket, 1u);
  }
  __syncthreads();
  int tile = s_ticket;
  if (tid < CW && tile < a.n_tiles) stage_params(sP, CW, coord_of(tile, a).cblk, tid, a);
  __syncthreads();
  uint32_t phase = 0;

  while (tile < a.n_tiles) {
    const TileCoord tc = coord_of(tile, a);
    const int c0 = tc.cblk * CW + g * V;
    const bool cvalid = c0 < R;
    const int t_start = tc.chunk * kScanTC + s * L;

    if (!mbar_wait(&bar, phase, &no_abort)) {
      if (tid == 0) atomicOr(a.status, kStatusTimeout);
    }
    // the ticket after `next` is fetched now; its round trip overlaps phase 1
    unsigned next2 = 0;
    if (tid == 0) next2 = atomicAdd(a.ticket, 1u);

    // ---- phase 1 ---------------------------------------------------------------------
    // Channels are taken four at a time, so that only four channels' parameters and
    // conv history are live at once.
    // Per-step replay values stay in registers: the shared-memory stage is refilled with the
    // next tile as soon as phase 1 is done.
    uint32_t rp[kAcc ? 1 : L * V];                    // bf16 path: (1 − a_t, b_t) pairs
    float ra[kAcc ? L * V : 1], rb[kAcc ? L * V : 1];  // f32 path: a_t, b_t
    float Ag[V], Bg[V];
    const bool from_state = (tc.chunk == 0 && s == 0 && a.state0 != nullptr);
#pragma unroll
    for (int vb = 0; vb < V; vb += 4) {
      const int cc = g * V + vb;  // channel offset inside the tile
      const float4 W0 = *reinterpret_cast<const float4*>(sP + 0 * CW + cc);
      const float4 W1 = *reinterpret_cast<const float4*>(sP + 1 * CW + cc);
      const float4 W2 = *reinterpret_cast<const float4*>(sP + 2 * CW + cc);
      const float4 W3 = *reinterpret_cast<const float4*>(sP + 3 * CW + cc);
      const float4 CB = *reinterpret_cast<const float4*>(sP + 4 * CW + cc);
      const float4 CL = *reinterpret_cast<const float4*>(sP + 5 * CW + cc);
      float4 xm3, xm2, xm1;
      if (from_state) {
        const T* st = static_cast<const T*>(a.state0) + (int64_t)tc.b * 3 * R + c0 + vb;
        xm3 = cvalid ? lds4<T>(st) : make_float4(0.f, 0.f, 0.f, 0.f);
        xm2 = cvalid ? lds4<T>(st + R) : make_float4(0.f, 0.f, 0.f, 0.f);
        xm1 = cvalid ? lds4<T>(st + 2 * R) : make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
        xm3 = lds4<T>(sx + (s * L + 0) * CW + cc);
        xm2 = lds4<T>(sx + (s * L + 1) * CW + cc);
        xm1 = lds4<T>(sx + (s * L + 2) * CW + cc);
      }
      float4 A4 = make_float4(1.f, 1.f, 1.f, 1.f), B4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int l = 0; l < L; ++l) {
        const int row = s * L + l;
        const float4 xc = lds4<T>(sx + (row + kHalo) * CW + cc);
        float4 za = lds4<T>(sza + row * CW + cc);
        const float4 zx = lds4<T>(szx + row * CW + cc);
        const bool tv = (t_start + l) < a.T;
        if (!kAcc && !tv) {
          // steps past T: r = σ(−∞) = 0 makes a_t = 1 and b_t = 0 (identity steps)
          za = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        }
        float2 u01 = __ffma2_rn(make_float2(W0.x, W0.y), make_float2(xm3.x, xm3.y), make_float2(CB.x, CB.y));
        float2 u23 = __ffma2_rn(make_float2(W0.z, W0.w), make_float2(xm3.z, xm3.w), make_float2(CB.z, CB.w));
        u01 = __ffma2_rn(make_float2(W1.x, W1.y), make_float2(xm2.x, xm2.y), u01);
        u23 = __ffma2_rn(make_float2(W1.z, W1.w), make_float2(xm2.z, xm2.w), u23);
        u01 = __ffma2_rn(make_float2(W2.x, W2.y), make_float2(xm1.x, xm1.y), u01);
        u23 = __ffma2_rn(make_float2(W2.z, W2.w), make_float2(xm1.z, xm1.w), u23);
        u01 = __ffma2_rn(make_float2(W3.x, W3.y), make_float2(xc.x, xc.y), u01);
        u23 = __ffma2_rn(make_float2(W3.z, W3.w), make_float2(xc.z, xc.w), u23);
        const float4 u = make_float4(u01.x, u01.y, u23.x, u23.y);
        float2 at0, bt0, at1, bt1;
        if constexpr (kAcc) {
          gate_accurate(za.x, zx.x, CL.x, u.x, at0.x, bt0.x);
          gate_accurate(za.y, zx.y, CL.y, u.y, at0.y, bt0.y);
          gate_accurate(za.z, zx.z, CL.z, u.z, at1.x, bt1.x);
          gate_accurate(za.w, zx.w, CL.w, u.w, at1.y, bt1.y);
          if (!tv) { at0 = at1 = make_float2(1.f, 1.f); bt0 = bt1 = make_float2(0.f, 0.f); }
          ra[l * V + vb + 0] = at0.x; ra[l * V + vb + 1] = at0.y; ra[l * V + vb + 2] = at1.x; ra[l * V + vb + 3] = at1.y;
          rb[l * V + vb + 0] = bt0.x; rb[l * V + vb + 1] = bt0.y; rb[l * V + vb + 2] = bt1.x; rb[l * V + vb + 3] = bt1.y;
        } else {
          float2 d0, d1;
          gate_fast2(make_float2(za.x, za.y), make_float2(zx.x, zx.y), make_float2(CL.x, CL.y),
                     make_float2(u.x, u.y), d0, bt0);
          gate_fast2(make_float2(za.z, za.w), make_float2(zx.z, zx.w), make_float2(CL.z, CL.w),
                     make_float2(u.z, u.w), d1, bt1);
          at0 = make_float2(1.f - d0.x, 1.f - d0.y);
          at1 = make_float2(1.f - d1.x, 1.f - d1.y);
          rp[l * V + vb + 0] = pack_bf16x2(d0.x, bt0.x);
          rp[l * V + vb + 1] = pack_bf16x2(d0.y, bt0.y);
          rp[l * V + vb + 2] = pack_bf16x2(d1.x, bt1.x);
          rp[l * V + vb + 3] = pack_bf16x2(d1.y, bt1.y);
        }
        // fold: (A, B) ← (a·A, a·B + b)
        const float2 B01 = __ffma2_rn(at0, make_float2(B4.x, B4.y), bt0);
        const float2 B23 = __ffma2_rn(at1, make_float2(B4.z, B4.w), bt1);
        const float2 A01 = __fmul2_rn(at0, make_float2(A4.x, A4.y));
        const float2 A23 = __fmul2_rn(at1, make_float2(A4.z, A4.w));
        A4 = make_float4(A01.x, A01.y, A23.x, A23.y);
        B4 = make_float4(B01.x, B01.y, B23.x, B23.y);
        xm3 = xm2;
        xm2 = xm1;
        xm1 = xc;
      }
      Ag[vb + 0] = A4.x; Ag[vb + 1] = A4.y; Ag[vb + 2] = A4.z; Ag[vb + 3] = A4.w;
      Bg[vb + 0] = B4.x; Bg[vb + 1] = B4.y; Bg[vb + 2] = B4.z; Bg[vb + 3] = B4.w;
    }
#pragma unroll
    for (int v = 0; v < V; v += 4) {
      *reinterpret_cast<float4*>(sA + s * CW + g * V + v) = make_float4(Ag[v], Ag[v + 1], Ag[v + 2], Ag[v + 3]);
      *reinterpret_cast<float4*>(sB + s * CW + g * V + v) = make_float4(Bg[v], Bg[v + 1], Bg[v + 2], Bg[v + 3]);
    }
    __syncthreads();
    // the x/z stage is free: prefetch the next tile
    const int next = s_next;
    __syncthreads();  // every thread has read s_next
    if (tid == 0) s_next = (int)next2;
    TileCoord nc{};
    if (next < a.n_tiles) nc = coord_of(next, a);
    if (tid == 0 && next < a.n_tiles) issue_tile_loads<T, kGate>(smem, &bar, maps, a, nc);

    // ---- phase 2 ---------------------------------------------------------------------
    // sP is not read after phase 1: the threads the look-back leaves idle stage the next
    // tile's parameters meanwhile
    if (tid >= CW && tid < 2 * CW && next < a.n_tiles && nc.cblk != tc.cblk)
      stage_params(sP, CW, nc.cblk, tid - CW, a);
    if (tid < CW) {
      const int j = tid;
      const int c = tc.cblk * CW + j;
      // exclusive prefixes (held in registers) map the tile's incoming state to the state
      // entering sub-chunk q
      float pA[S], pB[S];
#pragma unroll
      for (int q = 0; q < S; ++q) { pA[q] = sA[q * CW + j]; pB[q] = sB[q * CW + j]; }
      float A = 1.0f, Bv = 0.0f;
#pragma unroll
      for (int q = 0; q < S; ++q) {
        const float pa = pA[q], pb = pB[q];
        pA[q] = A;
        pB[q] = Bv;
        Bv = fmaf(pa, Bv, pb);
        A *= pa;
      }
      uint64_t* agg = a.carry_agg;
      uint32_t* incl = a.carry_incl;
      const bool publish = tc.tix != a.stall_tile;
      float hin;
      if (tc.chunk == 0) {
        hin = (a.h0 != nullptr && c < R) ? a.h0[(int64_t)tc.b * R + c] : 0.0f;
      } else {
        if (publish) st_relaxed_u64(agg + tc.tix * CW + j, ((uint64_t)__float_as_uint(Bv) << 32) | enc(A));
        // Walk back over earlier chunks of the same (b, channel block), composing their
        // aggregates until an inclusive state is found. (eA, eB) maps the state at the
        // end of chunk p to the state entering this tile.
        float eA = 1.0f, eB = 0.0f;
        int64_t p = tc.tix - 1;                      // nearest not yet composed predecessor
        const int64_t first = tc.tix - tc.chunk;     // chunk 0 of this (b, channel block)
        long long t0 = 0;
        while (true) {
          // one round trip reads the words of up to four predecessors p, p-1, p-2, p-3
          constexpr int kH = 4;
          uint32_t hw[kH];
          uint64_t aw[kH];
#pragma unroll
          for (int k = 0; k < kH; ++k) {
            const int64_t q = p - k;
            hw[k] = q >= first ? ld_relaxed_u32(incl + q * CW + j) : 0u;
            aw[k] = q >= first ? ld_relaxed_u64(agg + q * CW + j) : 0ull;
          }
          bool done = false;
          int used = 0;
#pragma unroll
          for (int k = 0; k < kH; ++k) {
            if (done || used != k || p - k < first) continue;
            if (hw[k] != 0u) {
              hin = fmaf(eA, dec(hw[k]), eB);
              done = true;
            } else if ((uint32_t)aw[k] != 0u) {  // the low half (A) is encoded; B is stored plainly
              eB = fmaf(eA, __uint_as_float((uint32_t)(aw[k] >> 32)), eB);
              eA *= dec((uint32_t)aw[k]);
              ++used;
            }
          }
          if (done) break;
          if (used > 0) {
            p -= used;
            t0 = 0;
            continue;
          }
          if (t0 == 0) {
            t0 = clock64();
          } else if (clock64() - t0 > kWaitCycles) {
            atomicOr(a.status, kStatusTimeout);
            hin = eB;
            break;
          }
        }
      }
      const float hout = fmaf(A, hin, Bv);
      if (publish) st_relaxed_u32(incl + tc.tix * CW + j, enc(hout));
      if (tc.chunk == a.n_chunks - 1 && a.hT != nullptr && c < R) a.hT[(int64_t)tc.b * R + c] = hout;
#pragma unroll
      for (int q = 0; q < S; ++q) sB[q * CW + j] = fmaf(pA[q], hin, pB[q]);
    }
    __syncthreads();

    // ---- phase 3: replay from the incoming state, write y ----------------------------
    if (cvalid) {
      float h[V];
#pragma unroll
      for (int v = 0; v < V; v += 4) {
        const float4 f = *reinterpret_cast<const float4*>(sB + s * CW + g * V + v);
        h[v] = f.x; h[v + 1] = f.y; h[v + 2] = f.z; h[v + 3] = f.w;
      }
      T* __restrict__ y = static_cast<T*>(a.y);
#pragma unroll
      for (int l = 0; l < L; ++l) {
        const int t = t_start + l;
        float o[V];
#pragma unroll
        for (int v = 0; v < V; v += 2) {
          float2 at, bt;
          if constexpr (kAcc) {
            at = make_float2(ra[l * V + v], ra[l * V + v + 1]);
            bt = make_float2(rb[l * V + v], rb[l * V + v + 1]);
          } else {
            const uint32_t p0 = rp[l * V + v], p1 = rp[l * V + v + 1];
            at = make_float2(1.0f - bf16lo(p0), 1.0f - bf16lo(p1));
            bt = make_float2(bf16hi(p0), bf16hi(p1));
          }
          const float2 h2 = __ffma2_rn(at, make_float2(h[v], h[v + 1]), bt);
          h[v] = h2.x;
          h[v + 1] = h2.y;
          o[v] = h2.x;
          o[v + 1] = h2.y;
        }
        if constexpr (kGate) {
          float gg[V];
          unpack_row<V>(*reinterpret_cast<const uint4*>(sg + (s * L + l) * CW + g * V), gg);
#pragma unroll
          for (int v = 0; v < V; ++v) o[v] *= gelu_exact(gg[v]);
        }
        if (t < a.T) __stcs(reinterpret_cast<uint4*>(y + ((int64_t)tc.b * a.T + t) * R + c0), pack_row<V>(o));
      }
    }
    __syncthreads();  // sB and (gated) sg are free
    if (tid == 0 && kGate && next < a.n_tiles) issue_gate_load<T, kGate>(smem, &bar, maps, nc);
    tile = next;
    phase ^= 1u;
  }
}

std::atomic<int64_t> g_stall_tile{-1};

template <typename T, bool kGate>
cudaError_t launch_typed(const ScanArgs& a, const ScanMaps& maps, cudaStream_t s) {
  using Ly = SmemLayout<T, kGate>;
  auto kern = rglru_scan_kernel<T, kGate>;
  static int occ[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (occ[dev] == 0) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Ly::kAlloc);
    if (e != cudaSuccess) return e;
    int nb = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, kScanThreads, Ly::kAlloc);
    if (e != cudaSuccess) return e;
    occ[dev] = nb > 0 ? nb : 1;
  }
  const int64_t grid = std::min<int64_t>(a.n_tiles, (int64_t)occ[dev] * num_sms());
  kern<<<(unsigned)grid, kScanThreads, Ly::kAlloc, s>>>(maps, a);
  return cudaGetLastError();
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
  L.off_agg = 256;
  L.off_incl = L.off_agg + (((size_t)L.n_tiles * cw * 8 + 255) / 256) * 256;
  L.bytes = L.off_incl + (((size_t)L.n_tiles * cw * 4 + 255) / 256) * 256;
  L.zero_bytes = L.bytes;
  return L;
}

void set_scan_stall(int64_t tile) { g_stall_tile.store(tile); }
int64_t scan_stall() { return g_stall_tile.load(); }

cudaError_t launch_scan(const ScanArgs& a_in, bool bf16, cudaStream_t s) {
  ScanArgs a = a_in;
  a.stall_tile = scan_stall();
  ScanMaps maps;
  const CUtensorMapDataType dt = bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const int es = bf16 ? 2 : 4;
  const int cw = scan_cw(bf16);
  {
    cuuint64_t dims[3] = {(cuuint64_t)a.R, (cuuint64_t)a.T, (cuuint64_t)a.B};
    cuuint64_t strides[2] = {(cuuint64_t)a.R * es, (cuuint64_t)a.T * a.R * es};
    cuuint32_t box[3] = {(cuuint32_t)cw, (cuuint32_t)kXRows, 1};
    if (!encode(&maps.x, dt, 3, a.x, dims, strides, box)) return cudaErrorInvalidValue;
    if (a.g != nullptr) {
      cuuint32_t gbox[3] = {(cuuint32_t)cw, (cuuint32_t)kScanTC, 1};
      if (!encode(&maps.g, dt, 3, a.g, dims, strides, gbox)) return cudaErrorInvalidValue;
    } else {
      maps.g = maps.x;
    }
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)a.pitch, (cuuint64_t)a.B * a.T};
    cuuint64_t strides[1] = {(cuuint64_t)a.pitch * es};
    cuuint32_t box[2] = {(cuuint32_t)cw, (cuuint32_t)kScanTC};
    if (!encode(&maps.z, dt, 2, a.z, dims, strides, box)) return cudaErrorInvalidValue;
  }
  const bool gate = a.g != nullptr;
  if (bf16) return gate ? launch_typed<__nv_bfloat16, true>(a, maps, s) : launch_typed<__nv_bfloat16, false>(a, maps, s);
  return gate ? launch_typed<float, true>(a, maps, s) : launch_typed<float, false>(a, maps, s);
}

}  // namespace rglru
