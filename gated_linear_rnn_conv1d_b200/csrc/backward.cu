// Backward of Conv1D(4) + RG-LRU for bf16 IO (float32 arithmetic).
//
// Math: reverse-mode differentiation of "Griffin：将门控线性循环与局部注意力混合以实现高效的
// 语言模型", §实门线性循环单元 (RG-LRU), Eq. (1)–(4) with the log-space decay of the paragraph
// after them, and of the Conv1D of §循环块. Per batch row and channel, with r = σ(z_a),
// i = σ(z_x), log a_t = r_t·c·log σ(Λ), m_t = √(1 − a_t²), h_t = a_t h_{t−1} + m_t i_t u_t and
// g_t = ∂ℓ/∂h_t (which takes ∂ℓ/∂y_t = dy_t at each step and a_{t+1} g_{t+1} from the next):
//   ∂a_t = g_t h_{t−1}, ∂m_t = g_t i_t u_t, ∂i_t = g_t m_t u_t, ∂u_t ⊃ g_t m_t i_t,
//   ∂log a_t·r_t = ∂a_t a_t r_t − ∂m_t a_t² (r_t/m_t)      (r/m → 0 as r → 0),
//   ∂z_a = ∂log a_t·r_t · c log σ(Λ) · (1 − r_t),  ∂z_x = ∂i_t i_t (1 − i_t),
//   ∂ℓ/∂(log σ(Λ)) = Σ ∂log a_t·r_t · c,  ∂Λ = that · σ(−Λ).
//
// The reverse recurrence g_t = dy_t + a_{t+1} g_{t+1} is linear in g, so it runs in kBwdTC-step
// chunks like the forward scan: each chunk folds itself into a map g_{t0} = P g_{t1} + Q
// (bwd_maps_kernel); a short sequential pass per (row, channel) hands every chunk the g
// entering it from the right (bwd_carries_kernel); each chunk then replays its steps with
// the gate gradients fused (bwd_grads_kernel). The linears' gradients are tensor-core GEMMs
// (gemm_tc.cu): ∂u ⊃ ∂z·[W_a; W_x] on a transposed copy of the weights made here, ∂W_a and
// ∂W_x = ∂zᵀu with ∂z and u read in place as MN-major operands; the Conv1D backward is its
// own kernel.
#include <cstdint>
#include <cuda_bf16.h>

#include "gate_math.cuh"
#include "kernels.cuh"

namespace rglru {

namespace {

constexpr int kBwdThreads = 128;  // threads per block; each thread takes 2 channels
constexpr int kBwdTC = 64;        // time steps per chunk of the reverse recurrence

__device__ __forceinline__ float2 ld_bf2(const __nv_bfloat16* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}
// read-only data of the kernel (lets the compiler move the load ahead of unrelated stores)
__device__ __forceinline__ float2 ld_bf2_nc(const __nv_bfloat16* p) {
  return __bfloat1622float2(__ldg(reinterpret_cast<const __nv_bfloat162*>(p)));
}
__device__ __forceinline__ void st_bf2(__nv_bfloat16* p, float a, float b) {
  *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b);
}
// Ask L2 for the line holding p, ahead of its load (holds no register while in flight)
__device__ __forceinline__ void pf_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }
constexpr int kPfAhead = 16;  // steps between a line's prefetch and its load (Conv1D backward)

// −expm1(x) for x ∈ (−0.25, 0] on a pair of lanes: the Taylor series of e^x − 1 about 0 to
// degree 7, −x (1 + x/2 + x²/6 + x³/24 + x⁴/120 + x⁵/720 + x⁶/5040) (the scalar form's
// terms, evaluated in the same order)
__device__ __forceinline__ float2 neg_expm1_small2(float2 x) {
  float2 p = __ffma2_rn(x, make_float2(1.0f / 5040.0f, 1.0f / 5040.0f), make_float2(1.0f / 720.0f, 1.0f / 720.0f));
  p = __ffma2_rn(p, x, make_float2(1.0f / 120.0f, 1.0f / 120.0f));
  p = __ffma2_rn(p, x, make_float2(1.0f / 24.0f, 1.0f / 24.0f));
  p = __ffma2_rn(p, x, make_float2(1.0f / 6.0f, 1.0f / 6.0f));
  p = __ffma2_rn(p, x, make_float2(0.5f, 0.5f));
  p = __ffma2_rn(p, x, make_float2(1.0f, 1.0f));
  return __fmul2_rn(make_float2(-x.x, -x.y), p);
}

// column of channel c's recurrence-gate pre-activation in a packed gate row
__device__ __forceinline__ int64_t zcol(int c) { return (int64_t)256 * (c / 128) + (c % 128); }

// a_t from z_a (with its bias) and c·log σ(Λ) (fast exponentials: the operands are bf16)
__device__ __forceinline__ float decay_of(float za, float cla) {
  const float r = rcp_approx(1.0f + ex2_approx(-za * kLog2e));
  return ex2_approx(r * cla * kLog2e);
}

struct BwdDims {
  int B, T, R, n_chunks;
  int64_t pitch;  // packed gate row
};

// Pass 1: the map g_{t0} = P·g_{t1} + Q of each chunk [t0, t1) of kBwdTC steps.
__global__ void __launch_bounds__(kBwdThreads) bwd_maps_kernel(const __nv_bfloat16* __restrict__ z,
                                                               const __nv_bfloat16* __restrict__ dy,
                                                               const float* __restrict__ Lambda, float* __restrict__ P,
                                                               float* __restrict__ Q, BwdDims d) {
  const int c = 2 * (blockIdx.x * kBwdThreads + threadIdx.x);
  if (c >= d.R) return;
  const int b = blockIdx.y / d.n_chunks, chunk = blockIdx.y % d.n_chunks;
  const int t0 = chunk * kBwdTC, t1 = min(t0 + kBwdTC, d.T);
  const float cl0 = decay_log_coeff(Lambda[c]), cl1 = decay_log_coeff(Lambda[c + 1]);
  const float2 cl2 = make_float2(cl0, cl1);
  const __nv_bfloat16* zb = z + (int64_t)b * d.T * d.pitch + zcol(c);
  const __nv_bfloat16* dyb = dy + (int64_t)b * d.T * d.R + c;
  float2 an = make_float2(1.0f, 1.0f);
  if (t1 < d.T) {
    const float2 za = ld_bf2(zb + (int64_t)t1 * d.pitch);
    an = make_float2(decay_of(za.x, cl0), decay_of(za.y, cl1));
  }
  float2 p = make_float2(1.0f, 1.0f), q = make_float2(0.0f, 0.0f);
  // eight steps at a time, their loads issued together ahead of the chain
  for (int tb = t1 - 1; tb >= t0; tb -= 8) {
    float2 gv[8], zv[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int t = tb - j;
      gv[j] = t >= t0 ? ld_bf2(dyb + (int64_t)t * d.R) : make_float2(0.f, 0.f);
      zv[j] = t >= t0 ? ld_bf2(zb + (int64_t)t * d.pitch) : make_float2(0.f, 0.f);
    }
    // both channels in packed f32x2 arithmetic (the same operations as decay_of per lane)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (tb - j < t0) break;
      p = __fmul2_rn(an, p);
      q = __ffma2_rn(an, q, gv[j]);
      const float2 na = __fmul2_rn(zv[j], make_float2(-kLog2e, -kLog2e));
      const float2 e = __fadd2_rn(make_float2(ex2_approx(na.x), ex2_approx(na.y)), make_float2(1.0f, 1.0f));
      const float2 l = __fmul2_rn(__fmul2_rn(make_float2(rcp_approx(e.x), rcp_approx(e.y)), cl2),
                                  make_float2(kLog2e, kLog2e));
      an = make_float2(ex2_approx(l.x), ex2_approx(l.y));
    }
  }
  const int64_t o = ((int64_t)b * d.n_chunks + chunk) * d.R + c;
  *reinterpret_cast<float2*>(P + o) = p;
  *reinterpret_cast<float2*>(Q + o) = q;
}

// Pass 2: per (row, channel), from the last chunk to the first, the g entering each chunk
// from the right (g_{t1}; dh_T for the last chunk).
__global__ void __launch_bounds__(kBwdThreads) bwd_carries_kernel(const float* __restrict__ P,
                                                                  const float* __restrict__ Q,
                                                                  const float* __restrict__ dh_T,
                                                                  float* __restrict__ gin, BwdDims d) {
  const int c = 2 * (blockIdx.x * kBwdThreads + threadIdx.x);
  if (c >= d.R) return;
  const int b = blockIdx.y;
  float2 G = dh_T != nullptr ? *reinterpret_cast<const float2*>(dh_T + (int64_t)b * d.R + c) : make_float2(0.f, 0.f);
#pragma unroll 8
  for (int chunk = d.n_chunks - 1; chunk >= 0; --chunk) {
    const int64_t o = ((int64_t)b * d.n_chunks + chunk) * d.R + c;
    *reinterpret_cast<float2*>(gin + o) = G;
    const float2 p = *reinterpret_cast<const float2*>(P + o), q = *reinterpret_cast<const float2*>(Q + o);
    G = make_float2(fmaf(p.x, G.x, q.x), fmaf(p.y, G.y, q.y));
  }
}

struct BwdGradArgs {
  const __nv_bfloat16* z;   // packed pre-activations (with biases) [B·T][pitch]
  const __nv_bfloat16* u;   // Conv1D output [B][T][R]
  const __nv_bfloat16* y;   // forward output = h_t [B][T][R]
  const __nv_bfloat16* dy;  // [B][T][R]
  const float* h0;          // [B][R] or null (zeros)
  const float* Lambda;      // [R]
  const float* gin;         // [B][n_chunks][R]
  __nv_bfloat16* dz;        // [B·T][2R]: ∂z_a in columns [0, R), ∂z_x in [R, 2R)
  float* du;                // [B][T][R] the direct term ∂ℓ/∂u_t ⊃ g m i
  float* dLsum;             // [R] Σ ∂log a·r·c (atomic)
  float* db_a;              // [R] (atomic)
  float* db_x;              // [R] (atomic)
  float* dh0;               // [B][R] or null
};

// Pass 3: each chunk replays its steps from the g entering it, with the gate gradients. Steps
// go in blocks of kGradBlock aligned to multiples of it, their loads issued together ahead of
// the chain (a block of 8 held 160 registers a thread and ran slower than single steps).
constexpr int kGradBlock = 2;
__global__ void __launch_bounds__(kBwdThreads) bwd_grads_kernel(BwdGradArgs a, BwdDims d) {
  const int c = 2 * (blockIdx.x * kBwdThreads + threadIdx.x);
  if (c >= d.R) return;
  const int b = blockIdx.y / d.n_chunks, chunk = blockIdx.y % d.n_chunks;
  const int t0 = chunk * kBwdTC, t1 = min(t0 + kBwdTC, d.T);
  const float cl[2] = {decay_log_coeff(a.Lambda[c]), decay_log_coeff(a.Lambda[c + 1])};
  const int64_t row0 = (int64_t)b * d.T;
  const __nv_bfloat16* zb = a.z + row0 * d.pitch + zcol(c);
  const float2 cl2 = make_float2(cl[0], cl[1]);
  float2 gn = *reinterpret_cast<const float2*>(a.gin + ((int64_t)b * d.n_chunks + chunk) * d.R + c);
  float2 an = make_float2(1.0f, 1.0f);
  if (t1 < d.T) {
    const float2 za = ld_bf2(zb + (int64_t)t1 * d.pitch);
    an = make_float2(decay_of(za.x, cl[0]), decay_of(za.y, cl[1]));
  }
  const float2 h0v =
      a.h0 != nullptr ? *reinterpret_cast<const float2*>(a.h0 + (int64_t)b * d.R + c) : make_float2(0.f, 0.f);
  float2 sL = make_float2(0.f, 0.f), sa = make_float2(0.f, 0.f), sx = make_float2(0.f, 0.f);
  // this thread's elements at step tb of a block, walked back by pointer decrements
  const int64_t R = d.R, R2 = 2 * d.R, pitch = d.pitch;
  int tb = (t1 - 1) & ~(kGradBlock - 1);
  const __nv_bfloat16* p_dy = a.dy + (row0 + tb) * R + c;
  const __nv_bfloat16* p_u = a.u + (row0 + tb) * R + c;
  const __nv_bfloat16* p_y = a.y + (row0 + tb - 1) * R + c;  // h_{t−1} (read only for t > 0)
  const __nv_bfloat16* p_z = zb + (int64_t)tb * pitch;
  __nv_bfloat16* p_dz = a.dz + (row0 + tb) * R2 + c;
  float* p_du = a.du + (row0 + tb) * R + c;
  for (; tb >= t0; tb -= kGradBlock) {
    // steps tb … tb + kGradBlock − 1 of this chunk (those < t1), replayed from the last
    const int j_hi = min(kGradBlock - 1, t1 - 1 - tb);
    float2 dyv[kGradBlock], uv[kGradBlock], zav[kGradBlock], zxv[kGradBlock], hpv[kGradBlock];
#pragma unroll
    for (int j = 0; j < kGradBlock; ++j) {
      if (j <= j_hi) {
        dyv[j] = ld_bf2_nc(p_dy + j * R);
        uv[j] = ld_bf2_nc(p_u + j * R);
        zav[j] = ld_bf2_nc(p_z + j * pitch);
        zxv[j] = ld_bf2_nc(p_z + j * pitch + 128);
        hpv[j] = tb + j > 0 ? ld_bf2_nc(p_y + j * R) : h0v;
      }
    }
#pragma unroll
    for (int j = kGradBlock - 1; j >= 0; --j) {
      if (j > j_hi) continue;
      // both channels at once in packed f32x2 arithmetic (the hardware ex2/rcp/rsqrt per
      // lane): gates and decay as the forward's fast path, 1 − a_t² from the Taylor form of
      // −expm1 near 0
      const float2 one = make_float2(1.0f, 1.0f);
      const float2 g = __ffma2_rn(an, gn, dyv[j]);
      const float2 na = __fmul2_rn(zav[j], make_float2(-kLog2e, -kLog2e));
      const float2 nx = __fmul2_rn(zxv[j], make_float2(-kLog2e, -kLog2e));
      const float2 ea = __fadd2_rn(make_float2(ex2_approx(na.x), ex2_approx(na.y)), one);
      const float2 ex = __fadd2_rn(make_float2(ex2_approx(nx.x), ex2_approx(nx.y)), one);
      const float2 r = make_float2(rcp_approx(ea.x), rcp_approx(ea.y));
      const float2 i = make_float2(rcp_approx(ex.x), rcp_approx(ex.y));
      const float2 la = __fmul2_rn(r, cl2);
      const float2 l2 = __fmul2_rn(la, make_float2(kLog2e, kLog2e));
      const float2 at = make_float2(ex2_approx(l2.x), ex2_approx(l2.y));
      const float2 x2 = __fadd2_rn(la, la);
      const float2 qs = neg_expm1_small2(x2);
      const float2 ql = __ffma2_rn(make_float2(-at.x, -at.y), at, one);
      const float2 q = make_float2(x2.x > -0.25f ? qs.x : ql.x, x2.y > -0.25f ? qs.y : ql.y);  // 1 − a_t²
      const float2 rs = make_float2(rsqrt_approx(fmaxf(q.x, 1e-30f)), rsqrt_approx(fmaxf(q.y, 1e-30f)));
      const float2 qr = __fmul2_rn(q, rs), rr = __fmul2_rn(r, rs);
      const float2 mt = make_float2(q.x > 0.0f ? qr.x : 0.0f, q.y > 0.0f ? qr.y : 0.0f);        // √(1 − a_t²)
      const float2 r_over_m = make_float2(q.x > 0.0f ? rr.x : 0.0f, q.y > 0.0f ? rr.y : 0.0f);  // r / √(1 − a_t²)
      const float2 d_a = __fmul2_rn(g, hpv[j]);
      const float2 d_m = __fmul2_rn(__fmul2_rn(g, i), uv[j]);
      const float2 gm = __fmul2_rn(g, mt);
      const float2 d_i = __fmul2_rn(gm, uv[j]);
      const float2 dud = __fmul2_rn(gm, i);
      // ∂log a_t · r_t = ∂a_t a_t r_t − ∂m_t a_t² (r_t / m_t)
      const float2 t_a = __fmul2_rn(__fmul2_rn(d_a, at), r);
      const float2 t_m = __fmul2_rn(__fmul2_rn(d_m, at), at);
      const float2 dlr = __ffma2_rn(make_float2(-t_m.x, -t_m.y), r_over_m, t_a);
      const float2 dza = __fmul2_rn(__fmul2_rn(dlr, cl2), __fadd2_rn(one, make_float2(-r.x, -r.y)));
      const float2 dzx = __fmul2_rn(__fmul2_rn(d_i, i), __fadd2_rn(one, make_float2(-i.x, -i.y)));
      sL = __ffma2_rn(dlr, make_float2(kDecayC, kDecayC), sL);
      sa = __fadd2_rn(sa, dza);
      sx = __fadd2_rn(sx, dzx);
      gn = g;
      an = at;
      st_bf2(p_dz + j * R2, dza.x, dza.y);
      st_bf2(p_dz + j * R2 + R, dzx.x, dzx.y);
      *reinterpret_cast<float2*>(p_du + j * R) = dud;
    }
    p_dy -= kGradBlock * R;
    p_u -= kGradBlock * R;
    p_y -= kGradBlock * R;
    p_z -= kGradBlock * pitch;
    p_dz -= kGradBlock * R2;
    p_du -= kGradBlock * R;
  }
  if (chunk == 0 && a.dh0 != nullptr)  // the gradient reaching h_{−1} = h0
    *reinterpret_cast<float2*>(a.dh0 + (int64_t)b * d.R + c) = make_float2(an.x * gn.x, an.y * gn.y);
  atomicAdd(a.dLsum + c, sL.x);
  atomicAdd(a.dLsum + c + 1, sL.y);
  atomicAdd(a.db_a + c, sa.x);
  atomicAdd(a.db_a + c + 1, sa.y);
  atomicAdd(a.db_x + c, sx.x);
  atomicAdd(a.db_x + c + 1, sx.y);
}

// ∂Λ = ∂ℓ/∂(log σ(Λ)) · σ(−Λ), since log σ(Λ) = −log(1 + e^{−Λ}).
__global__ void bwd_lambda_kernel(const float* __restrict__ dLsum, const float* __restrict__ Lambda,
                                  float* __restrict__ dLambda, int R) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c < R) dLambda[c] = dLsum[c] / (1.0f + expf(Lambda[c]));
}

struct BwdConvArgs {
  const __nv_bfloat16* x;       // [B][T][R]
  const __nv_bfloat16* state0;  // [B][3][R] (x_{−3}, x_{−2}, x_{−1}) or null
  const float* conv_w;          // [4][R]
  const float* du;              // [B][T][R] ∂ℓ/∂u (direct and gate terms)
  __nv_bfloat16* dx;            // [B][T][R]
  __nv_bfloat16* dstate0;       // [B][3][R] or null
  float* dconv_w;               // [4][R] (atomic)
  float* dconv_b;               // [R] (atomic)
};

// Conv1D backward, u_t = b + Σ_k w_k x_{t−3+k}: dx_s = Σ_k w_k du_{s+3−k} (t < T),
// dw_k = Σ du_t x_{t−3+k}, db = Σ du_t; for the first chunk also the conv history's gradient.
__global__ void __launch_bounds__(kBwdThreads) bwd_conv_kernel(BwdConvArgs a, BwdDims d) {
  const int c = 2 * (blockIdx.x * kBwdThreads + threadIdx.x);
  if (c >= d.R) return;
  const int b = blockIdx.y / d.n_chunks, chunk = blockIdx.y % d.n_chunks;
  const int t0 = chunk * kBwdTC, t1 = min(t0 + kBwdTC, d.T);
  const int64_t base = (int64_t)b * d.T * d.R + c;
  float w[4][2];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 wk = *reinterpret_cast<const float2*>(a.conv_w + k * d.R + c);
    w[k][0] = wk.x;
    w[k][1] = wk.y;
  }
  auto du_at = [&](int t) -> float2 {  // total ∂ℓ/∂u_t, zero past T
    if (t >= d.T) return make_float2(0.f, 0.f);
    return *reinterpret_cast<const float2*>(a.du + base + (int64_t)t * d.R);
  };
  auto x_at = [&](int t) -> float2 {  // x_t, from the conv history for t < 0
    if (t >= 0) return ld_bf2(a.x + base + (int64_t)t * d.R);
    if (a.state0 == nullptr) return make_float2(0.f, 0.f);
    return ld_bf2(a.state0 + ((int64_t)b * 3 + (t + 3)) * d.R + c);
  };
  // sliding windows: du_{t..t+3} and x_{t−3..t}
  float2 dwin[4], xwin[4];
  for (int j = 0; j < 4; ++j) dwin[j] = du_at(t0 + j);
  for (int j = 0; j < 3; ++j) xwin[j] = x_at(t0 - 3 + j);
  float sw[4][2] = {}, sb[2] = {0.f, 0.f};
  // eight steps at a time: their x and the ∂u entering the window loaded together first
  for (int tb = t0; tb < t1; tb += 8) {
    float2 xb[8], db[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int tp = tb + kPfAhead + j;
      if (tp < t1) pf_l2(a.x + base + (int64_t)tp * d.R);
      if (tp + 4 < d.T && tp < t1) pf_l2(a.du + base + (int64_t)(tp + 4) * d.R);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      xb[j] = tb + j < t1 ? x_at(tb + j) : make_float2(0.f, 0.f);
      db[j] = tb + j < t1 ? du_at(tb + j + 4) : make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const int t = tb + jj;
      if (t >= t1) break;
      xwin[3] = xb[jj];
      float dxv[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float dut = j ? dwin[0].y : dwin[0].x;
        float acc = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) acc = fmaf(w[k][j], j ? dwin[3 - k].y : dwin[3 - k].x, acc);
        dxv[j] = acc;
#pragma unroll
        for (int k = 0; k < 4; ++k) sw[k][j] = fmaf(dut, j ? xwin[k].y : xwin[k].x, sw[k][j]);
        sb[j] += dut;
      }
      st_bf2(a.dx + base + (int64_t)t * d.R, dxv[0], dxv[1]);
      for (int j = 0; j < 3; ++j) { dwin[j] = dwin[j + 1]; xwin[j] = xwin[j + 1]; }
      dwin[3] = db[jj];
    }
  }
  if (chunk == 0 && a.dstate0 != nullptr) {
    // history slot s = 0, 1, 2 holds x_{s−3}: its gradient is Σ_k w_k du_{s−k}, 0 ≤ s−k < T
    for (int s = 0; s < 3; ++s) {
      float acc[2] = {0.f, 0.f};
      for (int k = 0; k <= s; ++k) {
        const float2 dv = du_at(s - k);
        acc[0] = fmaf(w[k][0], dv.x, acc[0]);
        acc[1] = fmaf(w[k][1], dv.y, acc[1]);
      }
      st_bf2(a.dstate0 + ((int64_t)b * 3 + s) * d.R + c, acc[0], acc[1]);
    }
  }
#pragma unroll
  for (int j = 0; j < 2; ++j) {
#pragma unroll
    for (int k = 0; k < 4; ++k) atomicAdd(a.dconv_w + k * d.R + c + j, sw[k][j]);
    atomicAdd(a.dconv_b + c + j, sb[j]);
  }
}

// out[j][i] = in[i][j] for a rows × cols bf16 matrix (leading dimensions ld_in, ld_out);
// columns rows..rows_pad−1 of out are written as zeros. 64 × 64 tiles through shared
// memory with 16-byte loads and stores: cols, ld_in, ld_out and rows_pad are multiples of 8
// and both pointers 16-byte aligned.
__global__ void __launch_bounds__(256) transpose_bf16_kernel(const __nv_bfloat16* __restrict__ in,
                                                             __nv_bfloat16* __restrict__ out, int64_t rows,
                                                             int64_t cols, int64_t ld_in, int64_t ld_out,
                                                             int64_t rows_pad) {
  __shared__ __align__(16) __nv_bfloat16 tile[64][72];  // rows padded to 144 bytes
  const int64_t r0 = (int64_t)blockIdx.y * 64, c0 = (int64_t)blockIdx.x * 64;
  for (int i = threadIdx.x; i < 512; i += 256) {
    const int rr = i / 8, cv = i % 8;
    const int64_t r = r0 + rr, c = c0 + cv * 8;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r < rows && c < cols) v = *reinterpret_cast<const uint4*>(in + r * ld_in + c);
    *reinterpret_cast<uint4*>(&tile[rr][cv * 8]) = v;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 512; i += 256) {
    const int cc = i / 8, rv = i % 8;
    const int64_t c = c0 + cc, r = r0 + rv * 8;
    if (c < cols && r < rows_pad) {
      uint32_t w[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const __nv_bfloat162 pr = __halves2bfloat162(tile[rv * 8 + 2 * q][cc], tile[rv * 8 + 2 * q + 1][cc]);
        w[q] = *reinterpret_cast<const uint32_t*>(&pr);
      }
      *reinterpret_cast<uint4*>(out + c * ld_out + r) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

cudaError_t transpose_bf16(const void* in, void* out, int64_t rows, int64_t cols, int64_t ld_in, int64_t ld_out,
                           int64_t rows_pad, cudaStream_t s) {
  if (cols % 8 || ld_in % 8 || ld_out % 8 || rows_pad % 8) return cudaErrorInvalidValue;
  const dim3 grid((unsigned)((cols + 63) / 64), (unsigned)((rows_pad + 63) / 64));
  if (grid.y > 65535u) return cudaErrorInvalidValue;
  transpose_bf16_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(in), static_cast<__nv_bfloat16*>(out),
                                              rows, cols, ld_in, ld_out, rows_pad);
  return cudaGetLastError();
}

}  // namespace

BwdLayout bwd_layout(int B, int T, int R) {
  BwdLayout L;
  const int64_t n = (int64_t)B * T;
  const int n_chunks = (T + kBwdTC - 1) / kBwdTC;
  auto r256 = [](size_t v) { return (v + 255) / 256 * 256; };
  size_t o = 256;  // status word
  L.off_u = o;      o += r256((size_t)n * R * 2);
  L.off_z = o;      o += r256((size_t)n * gate_pitch(R) * 2);
  L.off_P = o;      o += r256((size_t)B * n_chunks * R * 4);
  L.off_Q = o;      o += r256((size_t)B * n_chunks * R * 4);
  L.off_gin = o;    o += r256((size_t)B * n_chunks * R * 4);
  L.off_dz = o;     o += r256((size_t)n * 2 * R * 2);
  L.off_du = o;     o += r256((size_t)n * R * 4);
  L.off_wt = o;     o += r256((size_t)2 * R * R * 2);
  L.off_dL = o;     o += r256((size_t)R * 4);
  L.bytes = o;
  L.n_chunks = n_chunks;
  return L;
}

cudaError_t launch_backward(const BwdArgs& g, const BwdLayout& L, void* ws, cudaStream_t s) {
  uint8_t* w = static_cast<uint8_t*>(ws);
  unsigned* status = reinterpret_cast<unsigned*>(w);
  const int B = g.B, T = g.T, R = g.R;
  const int64_t n = (int64_t)B * T;
  void* u = w + L.off_u;
  void* z = g.z_saved != nullptr ? const_cast<void*>(g.z_saved) : static_cast<void*>(w + L.off_z);
  float* P = reinterpret_cast<float*>(w + L.off_P);
  float* Q = reinterpret_cast<float*>(w + L.off_Q);
  float* gin = reinterpret_cast<float*>(w + L.off_gin);
  __nv_bfloat16* dz = reinterpret_cast<__nv_bfloat16*>(w + L.off_dz);
  float* du = reinterpret_cast<float*>(w + L.off_du);
  __nv_bfloat16* wt = reinterpret_cast<__nv_bfloat16*>(w + L.off_wt);
  float* dLsum = reinterpret_cast<float*>(w + L.off_dL);
  cudaError_t e;
  // the accumulated outputs start at zero
  if ((e = cudaMemsetAsync(status, 0, 4, s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(dLsum, 0, (size_t)R * 4, s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(g.db_a, 0, (size_t)R * 4, s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(g.db_x, 0, (size_t)R * 4, s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(g.dconv_w, 0, (size_t)4 * R * 4, s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(g.dconv_b, 0, (size_t)R * 4, s)) != cudaSuccess) return e;
  // recompute u = Conv1D(x) and (unless the forward saved them) the packed pre-activations
  // z (with biases)
  if ((e = launch_conv1d(g.conv_w, g.conv_b, g.x, g.state0, u, nullptr, B, T, R, true, status, s)) != cudaSuccess)
    return e;
  if (g.z_saved == nullptr && (e = launch_gemm_gates_bf16(u, g.W_a, g.b_a, g.W_x, g.b_x, z, n, R, status, s)) !=
                                   cudaSuccess)
    return e;
  BwdDims d{B, T, R, L.n_chunks, gate_pitch(R)};
  const unsigned gx = (unsigned)((R / 2 + kBwdThreads - 1) / kBwdThreads);
  const dim3 g_chunks(gx, (unsigned)(B * L.n_chunks)), g_rows(gx, (unsigned)B);
  bwd_maps_kernel<<<g_chunks, kBwdThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(z),
                                                   static_cast<const __nv_bfloat16*>(g.dy), g.Lambda, P, Q, d);
  bwd_carries_kernel<<<g_rows, kBwdThreads, 0, s>>>(P, Q, g.dh_T, gin, d);
  BwdGradArgs ga{static_cast<const __nv_bfloat16*>(z), static_cast<const __nv_bfloat16*>(u),
                 static_cast<const __nv_bfloat16*>(g.y), static_cast<const __nv_bfloat16*>(g.dy), g.h0, g.Lambda, gin,
                 dz, du, dLsum, g.db_a, g.db_x, g.dh0};
  bwd_grads_kernel<<<g_chunks, kBwdThreads, 0, s>>>(ga, d);
  bwd_lambda_kernel<<<(R + 255) / 256, 256, 0, s>>>(dLsum, g.Lambda, g.dLambda, R);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // ∂ℓ/∂u ⊃ [∂z_a | ∂z_x]·[W_a; W_x], added in float32 to the direct term the gradient pass
  // wrote (∂u then reaches ∂x through the Conv1D backward without a rounding). The weights
  // are read in place (MN-major) when R is a multiple of 64, else through a transposed copy
  // [W_a; W_x]ᵀ = [R][2R].
  if (R % 64 == 0) {
    if ((e = launch_gemm_f32out_wcat(dz, g.W_a, g.W_x, du, n, R, R, R, true, status, s)) != cudaSuccess) return e;
  } else {
    if ((e = transpose_bf16(g.W_a, wt, R, R, R, 2 * R, R, s)) != cudaSuccess) return e;
    if ((e = transpose_bf16(g.W_x, wt + R, R, R, R, 2 * R, R, s)) != cudaSuccess) return e;
    if ((e = launch_gemm_f32out(dz, wt, du, n, R, 2 * R, R, true, status, s)) != cudaSuccess) return e;
  }
  // ∂W_a = ∂z_aᵀ u, ∂W_x = ∂z_xᵀ u over the tokens: ∂z and u read in place, token-major
  // (MN-major operands)
  if ((e = launch_gemm_f32out_mn(dz, 2 * R, u, R, g.dW_a, R, R, n, R, status, s)) != cudaSuccess) return e;
  if ((e = launch_gemm_f32out_mn(dz + R, 2 * R, u, R, g.dW_x, R, R, n, R, status, s)) != cudaSuccess) return e;
  // Conv1D backward
  BwdConvArgs ca{static_cast<const __nv_bfloat16*>(g.x), static_cast<const __nv_bfloat16*>(g.state0), g.conv_w, du,
                 static_cast<__nv_bfloat16*>(g.dx), static_cast<__nv_bfloat16*>(g.dstate0), g.dconv_w,
                 g.dconv_b};
  bwd_conv_kernel<<<g_chunks, kBwdThreads, 0, s>>>(ca, d);
  return cudaGetLastError();
}

}  // namespace rglru
