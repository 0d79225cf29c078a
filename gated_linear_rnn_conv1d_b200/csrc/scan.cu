// Fused RG-LRU scan: Conv1D recompute + σ gates + log-space decay + chunked diagonal
// recurrence, one HBM read of x and of the gate pre-activations, one write of y.
//
// Math: "Griffin：将门控线性循环与局部注意力混合以实现高效的语言模型",
// §实门线性循环单元 (RG-LRU), Eq. (1)–(4); §循环块 for the Conv1D and the GeLU branch.
// Parallelisation: the recurrence h_t = a_t h_{t-1} + b_t is linear in h (neither gate
// reads h_{t-1}), so a chunk of steps composes into one affine map h ↦ A h + B with
// (A₁,B₁) then (A₂,B₂) giving (A₂A₁, A₂B₁ + B₂). Chunks are scanned independently and
// their summaries passed along ("Griffin's Compromise: Combining Gated Linear Recurrence
// with Local Attention", §Hawk, "Parallel scan").
//
// Work decomposition. A CTA owns one batch row b, CW consecutive channels and
// kScanTC = 64 consecutive steps. Its 256 threads are 16 channel groups (16 bytes of
// channels each) × 16 sub-chunks of kScanL = 4 steps.
//   phase 1  each thread loads its rows (x with a 3-row halo for the conv, z_a, z_x),
//            forms a_t, b_t in registers and folds them into its sub-chunk's (A, B);
//   phase 2  one thread per channel scans the 16 sub-chunk summaries in shared memory,
//            then obtains the CTA's incoming state by decoupled look-back over the
//            preceding time chunks of the same (b, channel block): each CTA publishes
//            its aggregate as soon as it is known and its inclusive state once its
//            incoming state is known; waits are bounded (status bit on timeout);
//   phase 3  each thread replays its 4 steps from its incoming state, writing y.
// Tiles are handed out by an atomic ticket in time-chunk-major order, so every tile a
// CTA waits for belongs to a CTA that started earlier (forward progress).
#include <atomic>
#include <cstdint>
#include <cuda_bf16.h>

#include "gate_math.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace rglru {

namespace {

constexpr unsigned kFlagAggregate = 1u;
constexpr unsigned kFlagInclusive = 2u;
constexpr unsigned kFlagGaveUp = 3u;   // local marker only, never stored

template <typename T> struct Vec;
template <> struct Vec<__nv_bfloat16> {
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
template <> struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void unpack(const uint4& v, float (&f)[4]) {
    f[0] = __uint_as_float(v.x); f[1] = __uint_as_float(v.y); f[2] = __uint_as_float(v.z); f[3] = __uint_as_float(v.w);
  }
  __device__ static uint4 pack(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
  }
};

__device__ __forceinline__ uint4 ldg16(const void* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  return __ldcs(reinterpret_cast<const uint4*>(p));  // read once: evict-first
}
__device__ __forceinline__ void st_stream16(void* p, const uint4& v) { __stcs(reinterpret_cast<uint4*>(p), v); }

__device__ __forceinline__ void named_bar(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

template <typename T, bool kAccurate, bool kGate>
__global__ void __launch_bounds__(kScanThreads, 2) rglru_scan_kernel(const ScanArgs a) {
  constexpr int V = Vec<T>::N;
  constexpr int CW = kScanGroups * V;
  constexpr int S = kScanSub;
  constexpr int L = kScanL;

  __shared__ float sA[S][CW];
  __shared__ float sB[S][CW];
  __shared__ __align__(16) float sP[6][CW];
  __shared__ unsigned s_ticket;
  __shared__ unsigned s_flag;

  const int tid = threadIdx.x;
  if (tid == 0) s_ticket = atomicAdd(a.ticket, 1u);
  __syncthreads();
  const unsigned ticket = s_ticket;
  const int per_chunk = a.B * a.n_cblk;
  const int chunk = (int)(ticket / per_chunk);
  const int rem = (int)(ticket % per_chunk);
  const int b = rem / a.n_cblk;
  const int cblk = rem % a.n_cblk;
  const int64_t tix = ((int64_t)b * a.n_cblk + cblk) * a.n_chunks + chunk;

  const int g = tid % kScanGroups;       // channel group
  const int s = tid / kScanGroups;       // sub-chunk
  const int c0 = cblk * CW + g * V;      // first channel of this thread
  const bool cvalid = c0 < a.R;
  const int t_start = chunk * kScanTC + s * L;
  const int R = a.R;
  const T* __restrict__ x = static_cast<const T*>(a.x);
  const T* __restrict__ z = static_cast<const T*>(a.z);
  const int64_t zoff = (int64_t)(c0 / kGateBlock) * 2 * kGateBlock + (c0 % kGateBlock);

  // ---- phase 1: loads --------------------------------------------------------------
  uint4 xr[L + 3], zar[L], zxr[L], gr[kGate ? L : 1];
#pragma unroll
  for (int j = 0; j < L + 3; ++j) {
    const int t = t_start - 3 + j;
    xr[j] = make_uint4(0, 0, 0, 0);
    if (cvalid) {
      if (t >= 0 && t < a.T) {
        const T* p = x + ((int64_t)b * a.T + t) * R + c0;
        xr[j] = (j < 3) ? ldg16(p) : ld_stream16(p);
      } else if (t < 0 && a.state0 != nullptr) {
        xr[j] = ldg16(static_cast<const T*>(a.state0) + ((int64_t)b * 3 + (t + 3)) * R + c0);
      }
    }
  }
#pragma unroll
  for (int l = 0; l < L; ++l) {
    const int t = t_start + l;
    zar[l] = zxr[l] = make_uint4(0, 0, 0, 0);
    if constexpr (kGate) gr[l] = make_uint4(0, 0, 0, 0);
    if (cvalid && t < a.T) {
      const T* zrow = z + ((int64_t)b * a.T + t) * a.pitch + zoff;
      zar[l] = ld_stream16(zrow);
      zxr[l] = ld_stream16(zrow + kGateBlock);
      if constexpr (kGate) gr[l] = ld_stream16(static_cast<const T*>(a.g) + ((int64_t)b * a.T + t) * R + c0);
    }
  }

  // per-channel parameters, staged once per CTA in shared memory: conv taps 0..3,
  // conv bias, c·log σ(Λ)
  if (tid < CW) {
    const int c = cblk * CW + tid;
    const bool ok = c < R;
    sP[0][tid] = ok ? __ldg(a.conv_w + c) : 0.0f;
    sP[1][tid] = ok ? __ldg(a.conv_w + R + c) : 0.0f;
    sP[2][tid] = ok ? __ldg(a.conv_w + 2 * R + c) : 0.0f;
    sP[3][tid] = ok ? __ldg(a.conv_w + 3 * R + c) : 0.0f;
    sP[4][tid] = ok ? __ldg(a.conv_b + c) : 0.0f;
    sP[5][tid] = ok ? decay_log_coeff(__ldg(a.Lambda + c)) : 0.0f;
  }
  __syncthreads();

  // ---- phase 1: gates, decay, local fold -------------------------------------------
  float at[L][V], bt[L][V];
  float Ag[V], Bg[V];
  {
    float xm3[V], xm2[V], xm1[V];
    Vec<T>::unpack(xr[0], xm3);
    Vec<T>::unpack(xr[1], xm2);
    Vec<T>::unpack(xr[2], xm1);
#pragma unroll
    for (int v = 0; v < V; ++v) { Ag[v] = 1.0f; Bg[v] = 0.0f; }
#pragma unroll
    for (int l = 0; l < L; ++l) {
      float xc[V], za[V], zx[V];
      Vec<T>::unpack(xr[l + 3], xc);
      Vec<T>::unpack(zar[l], za);
      Vec<T>::unpack(zxr[l], zx);
      const bool tv = (t_start + l) < a.T;
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const int cc = g * V + v;
        float u = sP[4][cc];
        u = fmaf(sP[0][cc], xm3[v], u);
        u = fmaf(sP[1][cc], xm2[v], u);
        u = fmaf(sP[2][cc], xm1[v], u);
        u = fmaf(sP[3][cc], xc[v], u);
        float av, bv;
        gate<kAccurate>(za[v], zx[v], sP[5][cc], u, av, bv);
        if (!tv) { av = 1.0f; bv = 0.0f; }
        at[l][v] = av;
        bt[l][v] = bv;
        Bg[v] = fmaf(av, Bg[v], bv);
        Ag[v] *= av;
        xm3[v] = xm2[v];
        xm2[v] = xm1[v];
        xm1[v] = xc[v];
      }
    }
  }
#pragma unroll
  for (int v = 0; v < V; ++v) {
    sA[s][g * V + v] = Ag[v];
    sB[s][g * V + v] = Bg[v];
  }
  __syncthreads();

  // ---- phase 2: sub-chunk prefix, look-back across CTAs ---------------------------
  if (tid < CW) {
    const int j = tid;
    const int c = cblk * CW + j;
    float A = 1.0f, Bv = 0.0f;
#pragma unroll
    for (int q = 0; q < S; ++q) {
      const float pa = sA[q][j], pb = sB[q][j];
      sA[q][j] = A;                // exclusive prefix (maps the CTA's incoming state to
      sB[q][j] = Bv;               // the state entering sub-chunk q)
      Bv = fmaf(pa, Bv, pb);
      A *= pa;
    }
    float* carry = a.carry + tix * 3 * CW;
    float hin;
    if (chunk == 0) {
      hin = (a.h0 != nullptr && c < R) ? a.h0[(int64_t)b * R + c] : 0.0f;
    } else {
      carry[j] = A;
      carry[CW + j] = Bv;
      __threadfence();
      named_bar(1, CW);
      if (j == 0 && tix != a.stall_tile) st_release_u32(a.flags + tix, kFlagAggregate);
      // Walk back over earlier chunks of the same (b, channel block), composing the
      // aggregates until an inclusive state is found. E maps the state at the end of
      // the current predecessor to the state entering this CTA.
      float eA = 1.0f, eB = 0.0f;
      int64_t ptix = tix - 1;
      while (true) {
        if (j == 0) {
          unsigned f = ld_acquire_u32(a.flags + ptix);
          if (f == 0u) {
            const long long t0 = clock64();
            while ((f = ld_acquire_u32(a.flags + ptix)) == 0u) {
              if (clock64() - t0 > kWaitCycles) { f = kFlagGaveUp; atomicOr(a.status, kStatusTimeout); break; }
              __nanosleep(64);
            }
          }
          s_flag = f;
        }
        named_bar(1, CW);
        const unsigned f = s_flag;
        named_bar(1, CW);
        if (f == kFlagGaveUp) { hin = eB; break; }
        (void)ld_acquire_u32(a.flags + ptix);   // per-thread acquire before reading the carry
        const float* pc = a.carry + ptix * 3 * CW;
        if (f == kFlagInclusive) { hin = fmaf(eA, __ldcg(pc + 2 * CW + j), eB); break; }
        const float pa = __ldcg(pc + j), pb = __ldcg(pc + CW + j);
        eB = fmaf(eA, pb, eB);
        eA *= pa;
        --ptix;
      }
    }
    carry[2 * CW + j] = fmaf(A, hin, Bv);
    __threadfence();
    named_bar(1, CW);
    if (j == 0 && tix != a.stall_tile) st_release_u32(a.flags + tix, kFlagInclusive);
#pragma unroll
    for (int q = 0; q < S; ++q) sB[q][j] = fmaf(sA[q][j], hin, sB[q][j]);
  }
  __syncthreads();

  // ---- phase 3: replay from the incoming state, write y (and h_T) ------------------
  if (!cvalid) return;
  float h[V];
#pragma unroll
  for (int v = 0; v < V; ++v) h[v] = sB[s][g * V + v];
  T* __restrict__ y = static_cast<T*>(a.y);
#pragma unroll
  for (int l = 0; l < L; ++l) {
    const int t = t_start + l;
    float gg[V];
    if constexpr (kGate) Vec<T>::unpack(gr[l], gg);
    float o[V];
#pragma unroll
    for (int v = 0; v < V; ++v) {
      h[v] = fmaf(at[l][v], h[v], bt[l][v]);
      if constexpr (kGate) o[v] = h[v] * gelu_exact(gg[v]);
      else o[v] = h[v];
    }
    if (t < a.T) {
      st_stream16(y + ((int64_t)b * a.T + t) * R + c0, Vec<T>::pack(o));
      if (t == a.T - 1 && a.hT != nullptr) {
#pragma unroll
        for (int v = 0; v < V; ++v) a.hT[(int64_t)b * R + c0 + v] = h[v];
      }
    }
  }
}

}  // namespace

ScanLayout scan_layout(int B, int T, int R, bool bf16) {
  ScanLayout L;
  const int cw = scan_cw(bf16);
  L.n_cblk = (R + cw - 1) / cw;
  L.n_chunks = (T + kScanTC - 1) / kScanTC;
  L.n_tiles = (int64_t)B * L.n_cblk * L.n_chunks;
  L.off_flags = 256;
  L.off_carry = L.off_flags + (((size_t)L.n_tiles * 4 + 255) / 256) * 256;
  L.bytes = L.off_carry + (size_t)L.n_tiles * 3 * cw * sizeof(float);
  return L;
}

namespace {
std::atomic<int64_t> g_stall_tile{-1};
}
void set_scan_stall(int64_t tile) { g_stall_tile.store(tile); }
int64_t scan_stall() { return g_stall_tile.load(); }

cudaError_t launch_scan(const ScanArgs& a_in, bool bf16, cudaStream_t s) {
  ScanArgs a = a_in;
  a.stall_tile = scan_stall();
  const int64_t n_tiles = (int64_t)a.B * a.n_cblk * a.n_chunks;
  dim3 grid((unsigned)n_tiles), block(kScanThreads);
  const bool gate = a.g != nullptr;
  if (bf16) {
    if (gate) rglru_scan_kernel<__nv_bfloat16, false, true><<<grid, block, 0, s>>>(a);
    else rglru_scan_kernel<__nv_bfloat16, false, false><<<grid, block, 0, s>>>(a);
  } else {
    if (gate) rglru_scan_kernel<float, true, true><<<grid, block, 0, s>>>(a);
    else rglru_scan_kernel<float, true, false><<<grid, block, 0, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace rglru
