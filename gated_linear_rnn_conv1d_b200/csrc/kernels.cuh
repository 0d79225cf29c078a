// Launch interfaces of the RG-LRU kernels (host side), shared by the C-ABI layer.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace rglru {

// ---- packed gate layout: 128-channel blocks, [z_a(128) | z_x(128)] per block -----
constexpr int kGateBlock = 128;
inline int64_t gate_pitch(int R) { return (int64_t)((R + kGateBlock - 1) / kGateBlock) * 2 * kGateBlock; }

// ---- scan tiling -------------------------------------------------------------------
constexpr int kScanTC = 64;   // time steps per tile (one chunk)
constexpr int kScanSub = 16;  // sub-chunks per tile
inline int scan_cw(bool bf16) { return bf16 ? 128 : 64; }  // channels per tile

struct ScanLayout {
  int n_cblk, n_chunks;
  int64_t n_tiles;
  // workspace: [status u32 | ticket u32 | pad to 256 B][inclusive states: n_tiles × CW × u32]
  // [aggregates: n_tiles × CW × u64]; all of it must be zero at launch
  size_t off_incl, off_agg, bytes, zero_bytes;
};
ScanLayout scan_layout(int B, int T, int R, bool bf16);

// TMA tensor maps the scan reads its tiles through.
struct ScanMaps {
  CUtensorMap x;  // [B][T][R], box {CW, 67, 1} (not encoded for the coefficient scan)
  CUtensorMap z;  // [B·T][pitch], box {CW, 64}
};

struct ScanArgs {
  const void* x;        // [B][T][R]
  const void* z;        // [B*T][pitch] packed
  const void* state0;   // [B][3][R] or null
  const float* h0;      // [B][R] or null
  const void* g;        // [B][T][R] or null (block gate branch)
  void* y;              // [B][T][R]
  float* hT;            // [B][R] or null
  const float* conv_w;  // [4][R]
  const float* conv_b;  // [R]
  const float* Lambda;  // [R]
  unsigned* status;     // device status word
  unsigned* ticket;     // tile ticket counter (zero at launch)
  uint32_t* carry_incl; // [n_tiles][CW] published inclusive states (zero at launch)
  uint64_t* carry_agg;  // [n_tiles][CW] published tile maps (A, B) (zero at launch)
  int B, T, R, n_cblk, n_chunks, n_tiles;
  int64_t pitch;
  int64_t stall_tile;   // testing only: this tile never publishes its carry (-1: none)
};
// Testing only: the tile index the next scans leave unpublished (-1 disables).
void set_scan_stall(int64_t tile);
int64_t scan_stall();
// coef: z holds the recurrence coefficients (d = 1 − a_t fp16, b_t = √(1−a_t²)·i_t·u_t bf16)
// that launch_gemm_coeffs_bf16 forms, instead of pre-activations (bf16 IO only); x, the
// conv parameters and Λ are then not read.
cudaError_t launch_scan(const ScanArgs& a, bool bf16, cudaStream_t s, bool coef = false);

// ---- conv --------------------------------------------------------------------------
// zero/zero_bytes (16-byte aligned, a multiple of 16): a region the kernel also zeroes (the
// scan workspace of the same forward), or none.
cudaError_t launch_conv1d(const float* conv_w, const float* conv_b, const void* x, const void* state0, void* u,
                          void* stateT, int B, int T, int R, bool bf16, unsigned* status, cudaStream_t s,
                          void* zero = nullptr, size_t zero_bytes = 0);
// Also zeroes *status (the step's status word) before the step's GEMM may set it.
cudaError_t launch_decode_conv(const float* conv_w, const float* conv_b, const float* Lambda, const void* x_t,
                               void* ring, int64_t step, void* u_t, float* u_f32, float* cla, unsigned* status,
                               int B, int R, cudaStream_t s);

// ---- GEMMs -------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn get_encode_tiled();
int num_sms();

// `status`: device word the kernel ORs kStatusTimeout into if a bounded wait gives up.
// The gate GEMM with the recurrence coefficients formed in its epilogue: g packed like z,
// d = 1 − a_t (fp16) in the z_a places and b_t = √(1−a_t²)·i_t·u_t (bf16) in the z_x places (the
// epilogue reads its rows of u, the GEMM's A operand).
// z_out, when not null, receives the pre-activations z in the packed layout of g (what
// launch_gemm_gates_bf16 writes, bit for bit).
cudaError_t launch_gemm_coeffs_bf16(const void* u, const void* Wa, const float* ba, const void* Wx, const float* bx,
                                    const float* Lambda, void* g, int64_t M, int R, unsigned* status, cudaStream_t s,
                                    void* z_out = nullptr);
cudaError_t launch_gemm_gates_bf16(const void* u, const void* Wa, const float* ba, const void* Wx, const float* bx,
                                   void* z, int64_t M, int R, unsigned* status, cudaStream_t s);
cudaError_t launch_gemm_bf16(const void* A, const void* Bm, void* C, int64_t M, int N, int K, int64_t ldc,
                             unsigned* status, cudaStream_t s);
// launch_gemm_bf16 for few output tiles (M a decode batch): K is split over about every SM
// pair, the slices' float32 partial sums go to `part` (at most kSplitPartBytes are used)
// and a second kernel sums them into C. Falls back to launch_gemm_bf16 when the output
// tiles alone fill the GPU or part is null.
constexpr size_t kSplitPartBytes = (size_t)80 * 256 * 256 * 4;
cudaError_t launch_gemm_bf16_skinny(const void* A, const void* Bm, void* C, int64_t M, int N, int K, int64_t ldc,
                                    float* part, size_t part_bytes, unsigned* status, cudaStream_t s);
// The split launch_gemm_bf16_skinny would choose (1: not split), and its GEMM alone: slice
// s of the K blocks writes its float32 partial sums to part + s·M·N ([M][N] each).
int skinny_splits(int64_t M, int N, int K, size_t part_bytes);
cudaError_t launch_gemm_partials(const void* A, const void* Bm, int64_t M, int N, int K, float* part, int ksp,
                                 unsigned* status, cudaStream_t s);
// C = A·Bᵀ (or C += A·Bᵀ with `accumulate`) as launch_gemm_bf16 (A [M][K], B [N][K] bf16,
// K-contiguous), C float32 [M][ldc], N a multiple of 4.
cudaError_t launch_gemm_f32out(const void* A, const void* Bm, float* C, int64_t M, int N, int K, int64_t ldc,
                               bool accumulate, unsigned* status, cudaStream_t s);
// C = Aᵀ·B, float32 C [M][ldc]: A [K][lda] (M columns) and B [K][ldb] (N columns) bf16 row-major,
// read in place as MN-major tensor-core operands (K = the reduction over rows, e.g. tokens).
// lda, ldb multiples of 8, A and B 16-byte aligned.
cudaError_t launch_gemm_f32out_mn(const void* A, int64_t lda, const void* Bm, int64_t ldb, float* C, int M, int N,
                                  int64_t K, int64_t ldc, unsigned* status, cudaStream_t s);
// C = A·[W0; W1] (or C += with `accumulate`), float32 C [M][ldc]: A [M][2·Kh] bf16 K-major,
// W0 and W1 [Kh][N] bf16 row-major (the stacked matrix's first and second Kh rows), read in
// place as an MN-major operand. Kh a multiple of 64, N of 8.
cudaError_t launch_gemm_f32out_wcat(const void* A, const void* W0, const void* W1, float* C, int64_t M, int N,
                                    int Kh, int64_t ldc, bool accumulate, unsigned* status, cudaStream_t s);
cudaError_t launch_gemm_step_bf16(const void* u_t, const float* u_f32, const void* Wa, const float* ba,
                                  const void* Wx, const float* bx, const float* cla, float* h, void* y_t, int B,
                                  int R, unsigned* status, cudaStream_t s);
// Gate GEMM (2-SM tcgen05) with the RG-LRU scan fused into its epilogue (bf16 IO,
// T % 128 == 0): y and h_T straight from x and u, without writing the gate
// pre-activations. carry_* need n_chunk_tiles × 128 slots (zero at launch).
struct ScanFusedArgs {
  const void* u;        // [B·T][R] bf16 conv output (GEMM operand, and the u of b_t)
  const void* W_a;
  const void* W_x;
  const float* b_a;
  const float* b_x;
  const float* Lambda;
  const float* h0;      // or null
  void* y;              // [B][T][R] bf16
  float* hT;            // or null
  uint64_t* carry_agg;  // [B · ceil(R/128) · T/128][128]
  uint32_t* carry_incl; // [B · ceil(R/128) · T/128][128]
  unsigned* status;
  int B, T, R;
};
cudaError_t launch_gate_scan_bf16(const ScanFusedArgs& f, cudaStream_t s);

// Library-global device status word of the current device (for entry points that take
// no workspace); null if the symbol address cannot be obtained.
unsigned* global_status_word();
cudaError_t launch_gemm_gates_f32(const float* u, const float* Wa, const float* ba, const float* Wx,
                                  const float* bx, float* z, int64_t M, int R, cudaStream_t s);

// ---- Hawk residual layer: elementwise kernels (bf16, 16-byte aligned, D % 8 == 0) ------
// y = x + o (skipped if o is null; y then unused) and n = RMSNorm(y or x) ⊙ scale (skipped
// if n is null) over rows of D channels; x, o, y, n distinct.
cudaError_t launch_add_rmsnorm(const void* x, const void* o, void* y, void* n, const float* scale, int64_t rows,
                               int D, float eps, cudaStream_t s);
// p = GeLU(gate) ⊙ up over n elements (n % 8 == 0); p may be gate.
cudaError_t launch_gelu_mul(const void* gate, const void* up, void* p, int64_t n, cudaStream_t s);

// ---- Griffin local multi-query attention, decode step (attention.cu) ----------------------
// D_head = 128, H = D / 128 query heads (1 ≤ H ≤ kAttnMaxHeads), one key/value head; the
// window W a multiple of 128. Workspace: [status word | qkv [B][(H+2)·128] bf16 | rotated
// queries [B][H][128] bf16 | partial outputs [B][W/128][H][128] f32 | maxima, sums
// [B][W/128][H] f32 | o [B][H·128] bf16 | the projections' split-K partial sums].
constexpr int kAttnMaxHeads = 64;
struct AttnLayout {
  int H, n_chunks;
  size_t off_qkv, off_q, off_op, off_m, off_l, off_o, off_part, bytes;
};
AttnLayout attn_layout(int B, int D, int W);
// RoPE and ring writes of position `pos` from the projection — qkv [B][(H+2)·128] bf16, or,
// when qkv_part is not null, the sum of its ksp float32 slices (rounded to bf16 first) —
// then the windowed attention into the workspace's o. k_ring, v_ring [B][W][128] bf16, in
// place.
cudaError_t launch_attention_core(const void* qkv, const float* qkv_part, int ksp, void* k_ring, void* v_ring,
                                  int64_t pos, int B, int D, int W, const AttnLayout& L, void* ws, unsigned* status,
                                  cudaStream_t s);

// ---- backward (bf16 IO) --------------------------------------------------------------
// Workspace of launch_backward: [status | u | z | chunk maps P, Q | chunk carries | ∂z |
// ∂u (f32: the direct term, then the gate GEMM's added) | [W_a; W_x]ᵀ | Σ ∂log a·r·c].
struct BwdLayout {
  size_t off_u, off_z, off_P, off_Q, off_gin, off_dz, off_du, off_wt, off_dL, bytes;
  int n_chunks;
};
BwdLayout bwd_layout(int B, int T, int R);
struct BwdArgs {
  const void* x;        // [B][T][R] bf16
  const void* y;        // forward output [B][T][R] bf16
  const void* dy;       // [B][T][R] bf16
  const float* h0;      // [B][R] or null
  const float* dh_T;    // [B][R] or null
  const void* state0;   // [B][3][R] bf16 or null
  const float* conv_w;  // [4][R]
  const float* conv_b;
  const void* W_a;      // [R][R] bf16
  const float* b_a;
  const void* W_x;
  const float* b_x;
  const float* Lambda;
  void* dx;             // [B][T][R] bf16
  void* dstate0;        // [B][3][R] bf16 or null
  float* dconv_w;       // [4][R]
  float* dconv_b;       // [R]
  float* dW_a;          // [R][R]
  float* db_a;
  float* dW_x;
  float* db_x;
  float* dLambda;
  float* dh0;           // [B][R] or null
  const void* z_saved;  // the forward's pre-activations [B·T][gate_pitch(R)] bf16, or null (recomputed)
  int B, T, R;
};
cudaError_t launch_backward(const BwdArgs& g, const BwdLayout& L, void* ws, cudaStream_t s);

}  // namespace rglru
