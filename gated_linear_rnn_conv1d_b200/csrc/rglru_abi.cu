// C ABI of librglru.so (declared in include/rglru.h): argument validation, workspace
// layout and the launch sequence of each entry point. Every argument check happens
// before the first CUDA call, so an invalid call returns without touching the device.
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>
#include <mutex>
#include <nvtx3/nvToolsExt.h>

#include "../../include/rglru.h"
#include "kernels.cuh"
#include "ptx.cuh"

using namespace rglru;

namespace {

thread_local int g_last_cuda_error = 0;

// NVTX range around one C-ABI call (a no-op unless a profiler attaches NVTX handling), so a
// timeline or an `ncu --nvtx` filter can group the kernels one call launches.
struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
  Range(const Range&) = delete;
  Range& operator=(const Range&) = delete;
};

constexpr int kMaxDevices = 64;

int fail_cuda(cudaError_t e) {
  g_last_cuda_error = (int)e;
  return RGLRU_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }
size_t round256(size_t n) { return (n + 255) / 256 * 256; }
size_t esize(int io) { return io == RGLRU_BF16 ? 2 : 4; }

bool valid_dtype(int io) { return io == RGLRU_F32 || io == RGLRU_BF16; }

// R: channels; limits keep every TMA dimension and every 32-bit grid index in range.
bool valid_R(int R) { return R >= 8 && R % 8 == 0 && R <= 65536; }
bool valid_tokens(int64_t B, int64_t T) {
  return B >= 1 && T >= 1 && B <= 65535 && B * T <= (int64_t)INT32_MAX;
}

// Checks that the current device is a B200-class part (compute capability 10.0).
int check_device() {
  static int cc[kMaxDevices] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e);
  if (dev < 0 || dev >= kMaxDevices) return RGLRU_ERR_DEVICE;
  if (cc[dev] == 0) {
    int major = 0, minor = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess) return fail_cuda(e);
    if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess) return fail_cuda(e);
    cc[dev] = major * 10 + minor;
  }
  return cc[dev] == 100 ? RGLRU_OK : RGLRU_ERR_DEVICE;
}

int check_params(const rglru_params* p) {
  if (p == nullptr || p->conv_w == nullptr || p->conv_b == nullptr || p->W_a == nullptr || p->b_a == nullptr ||
      p->W_x == nullptr || p->b_x == nullptr || p->Lambda == nullptr)
    return RGLRU_ERR_NULL;
  if (!aligned16(p->conv_w) || !aligned16(p->conv_b) || !aligned16(p->W_a) || !aligned16(p->b_a) ||
      !aligned16(p->W_x) || !aligned16(p->b_x) || !aligned16(p->Lambda))
    return RGLRU_ERR_ALIGN;
  return RGLRU_OK;
}

// ---- workspace layouts -------------------------------------------------------------
struct FwdLayout {
  ScanLayout scan;
  size_t off_u, off_z, bytes;
};
FwdLayout fwd_layout(int B, int T, int R, int io) {
  FwdLayout L;
  L.scan = scan_layout(B, T, R, io == RGLRU_BF16);
  const size_t ntok = (size_t)B * T;
  L.off_u = round256(L.scan.bytes);
  L.off_z = L.off_u + round256(ntok * R * esize(io));
  L.bytes = L.off_z + round256(ntok * (size_t)gate_pitch(R) * esize(io));
  return L;
}

// Forward through the fused gate-GEMM + scan kernel (bf16 IO, T % 128 == 0):
// [status, ticket | chunk aggregates | chunk inclusive states][u]. Carries are zeroed per call.
struct FusedLayout {
  int64_t n_chunk_tiles;
  size_t off_agg, off_incl, zero_bytes, off_u, bytes;
};
FusedLayout fused_layout(int B, int T, int R) {
  FusedLayout L;
  L.n_chunk_tiles = (int64_t)B * ((R + 127) / 128) * (T / 128);
  L.off_agg = 256;
  L.off_incl = L.off_agg + round256((size_t)L.n_chunk_tiles * 128 * 8);
  L.zero_bytes = L.off_incl + round256((size_t)L.n_chunk_tiles * 128 * 4);
  L.off_u = L.zero_bytes;
  L.bytes = L.off_u + round256((size_t)B * T * R * 2);
  return L;
}
// rglru_forward takes the fused gate GEMM + scan (2 launches: Conv1D, then the GEMM with the
// scan in its epilogue) for bf16 IO, T a multiple of 128 and R ≥ 4096: its epilogue (the
// gate math twice and the scan, per 128 × 128 tile) then hides behind the tile's MMAs
// (K = R); at R = 2048 it does not and the separate gate GEMM + scan is faster (B=8 T=2048
// R=2048: 306 µs fused against 254 µs; B=1 T=32768 R=4096: 1.73–1.76 ms against 1.88 ms).
bool fused_ok(int io, int T) { return io == RGLRU_BF16 && T % 128 == 0; }
bool fused_faster(int io, int T, int R) { return fused_ok(io, T) && R >= 4096; }

ScanFusedArgs fused_args(const rglru_params* p, const void* u, const float* h0, void* y, float* hT, int B, int T, int R,
                         const FusedLayout& L, void* ws) {
  ScanFusedArgs f{};
  f.u = u;
  f.W_a = p->W_a;
  f.W_x = p->W_x;
  f.b_a = p->b_a;
  f.b_x = p->b_x;
  f.Lambda = p->Lambda;
  f.h0 = h0;
  f.y = y;
  f.hT = hT;
  f.carry_agg = reinterpret_cast<uint64_t*>(static_cast<uint8_t*>(ws) + L.off_agg);
  f.carry_incl = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + L.off_incl);
  f.status = reinterpret_cast<unsigned*>(ws);
  f.B = B;
  f.T = T;
  f.R = R;
  return f;
}

struct BlockLayout {
  ScanLayout scan;
  size_t off_v, off_g, off_u, off_z, off_p, bytes;
};
BlockLayout block_layout(int B, int T, int R) {
  BlockLayout L;
  L.scan = scan_layout(B, T, R, true);
  const size_t ntok = (size_t)B * T;
  const size_t act = round256(ntok * R * 2);
  L.off_v = round256(L.scan.bytes);
  L.off_g = L.off_v + act;
  L.off_u = L.off_g + act;
  L.off_z = L.off_u + act;
  L.off_p = L.off_z + round256(ntok * (size_t)gate_pitch(R) * 2);
  L.bytes = L.off_p + act;
  return L;
}

struct StepLayout {
  size_t off_cla, off_u, off_uf, bytes;
};
StepLayout step_layout(int B, int R) {
  StepLayout L;
  L.off_cla = 256;
  L.off_u = L.off_cla + round256((size_t)R * 4);
  L.off_uf = L.off_u + round256((size_t)B * R * 2);
  L.bytes = L.off_uf + round256((size_t)B * R * 4);
  return L;
}

uint8_t* bytes(void* p) { return static_cast<uint8_t*>(p); }

// Local attention: D a multiple of 128 (H = D/128 heads of 128), 1 ≤ H ≤ kAttnMaxHeads;
// window a multiple of 128, at most 65536.
bool valid_attention(int B, int D, int window) {
  return B >= 1 && B <= 65535 && D >= 128 && D % 128 == 0 && D / 128 <= kAttnMaxHeads && window >= 128 &&
         window % 128 == 0 && window <= 65536;
}

// Griffin's local-attention residual layer, decode step: [the attention step's workspace
// (status word at 0) | n [B][D] | o [B][D] | residual [B][D] | gate, up [B][Hm]], bf16.
struct AttnLayerLayout {
  AttnLayout attn;
  size_t off_n, off_o, off_res, off_gate, off_up, bytes;
};
AttnLayerLayout attn_layer_layout(int B, int D, int Hm, int window) {
  AttnLayerLayout L;
  L.attn = attn_layout(B, D, window);
  const size_t row = round256((size_t)B * D * 2), hid = round256((size_t)B * Hm * 2);
  L.off_n = round256(L.attn.bytes);
  L.off_o = L.off_n + row;
  L.off_res = L.off_o + row;
  L.off_gate = L.off_res + row;
  L.off_up = L.off_gate + hid;
  L.bytes = L.off_up + hid;
  return L;
}

// x_t → out_t through the local-attention block: the fused q/k/v projection, RoPE, ring
// update and windowed attention, the output projection.
cudaError_t attention_sequence(const rglru_attention_weights* w, const void* x_t, void* k_ring, void* v_ring,
                               void* out_t, int B, int D, int window, int64_t pos, const AttnLayout& L, void* ws,
                               cudaStream_t s) {
  unsigned* status = reinterpret_cast<unsigned*>(ws);
  const int nqkv = (L.H + 2) * 128;
  void* qkv = bytes(ws) + L.off_qkv;
  float* part = reinterpret_cast<float*>(bytes(ws) + L.off_part);
  // the projection split over K at a decode batch: its slices are summed by the RoPE kernel
  const int ksp = skinny_splits(B, nqkv, D, kSplitPartBytes);
  cudaError_t e = ksp > 1 ? launch_gemm_partials(x_t, w->W_qkv, B, nqkv, D, part, ksp, status, s)
                          : launch_gemm_bf16(x_t, w->W_qkv, qkv, B, nqkv, D, nqkv, status, s);
  if (e == cudaSuccess)
    e = launch_attention_core(qkv, ksp > 1 ? part : nullptr, ksp, k_ring, v_ring, pos, B, D, window, L, ws, status,
                              s);
  if (e == cudaSuccess)
    e = launch_gemm_bf16_skinny(bytes(ws) + L.off_o, w->W_o, out_t, B, D, L.H * 128, D, part, kSplitPartBytes,
                                status, s);
  return e;
}

// Hawk residual layer: [recurrent block workspace (status word at 0) | n: RMSNorm output
// [B·T][D] (RMSNorm₁, then RMSNorm₂) | o: component output [B·T][D] (the block's, then
// the MLP's) | y: residual stream [B·T][D] | gate (then p) [B·T][H] | up [B·T][H]], bf16.
struct LayerLayout {
  BlockLayout block;
  size_t off_n, off_o, off_y, off_gate, off_up, bytes;
};
LayerLayout layer_layout(int B, int T, int D, int R, int H) {
  LayerLayout L;
  L.block = block_layout(B, T, R);
  const size_t ntok = (size_t)B * T;
  const size_t actD = round256(ntok * D * 2), actH = round256(ntok * H * 2);
  L.off_n = round256(L.block.bytes);
  L.off_o = L.off_n + actD;
  L.off_y = L.off_o + actD;
  L.off_gate = L.off_y + actD;
  L.off_up = L.off_gate + actH;
  L.bytes = L.off_up + actH;
  return L;
}

// Decode step of the layer: [step workspace (status word at 0, the decode conv's own word
// at 4) | n [B][D] | v [B][R] | g, then GeLU(g) ⊙ y [B][R] | y [B][R] | o [B][D] | residual
// stream [B][D] | gate (then p) [B][H] | up [B][H]], bf16.
struct LayerStepLayout {
  StepLayout step;
  size_t off_n, off_v, off_g, off_y, off_o, off_res, off_gate, off_up, bytes;
};
LayerStepLayout layer_step_layout(int B, int D, int R, int H) {
  LayerStepLayout L;
  L.step = step_layout(B, R);
  const size_t b = (size_t)B;
  L.off_n = round256(L.step.bytes);
  L.off_v = L.off_n + round256(b * D * 2);
  L.off_g = L.off_v + round256(b * R * 2);
  L.off_y = L.off_g + round256(b * R * 2);
  L.off_o = L.off_y + round256(b * R * 2);
  L.off_res = L.off_o + round256(b * D * 2);
  L.off_gate = L.off_res + round256(b * D * 2);
  L.off_up = L.off_gate + round256(b * H * 2);
  L.bytes = L.off_up + round256(b * H * 2);
  return L;
}

// The recurrent block (§循环块, Fig. 2(c)) after its status word is zeroed: the two
// D → D_RNN linears, Conv1D, the coefficient GEMM, the gated scan (p = h ⊙ GeLU(g)) and
// the D_RNN → D linear, queued on s with the block workspace layout L.
cudaError_t block_sequence(const rglru_params* params, const void* W_1, const void* W_2, const void* W_o,
                           const void* x, const float* h0, void* out, float* h_T, int B, int T, int D, int R,
                           const BlockLayout& L, void* workspace, cudaStream_t s) {
  const int64_t ntok = (int64_t)B * T;
  void* v = bytes(workspace) + L.off_v;
  void* g = bytes(workspace) + L.off_g;
  void* u = bytes(workspace) + L.off_u;
  void* z = bytes(workspace) + L.off_z;
  void* pbuf = bytes(workspace) + L.off_p;
  unsigned* status = reinterpret_cast<unsigned*>(workspace);
  cudaError_t e = launch_gemm_bf16(x, W_1, v, ntok, R, D, R, status, s);  // v = x W_1ᵀ
  if (e == cudaSuccess) e = launch_gemm_bf16(x, W_2, g, ntok, R, D, R, status, s);        // g = x W_2ᵀ
  if (e == cudaSuccess)
    e = launch_conv1d(params->conv_w, params->conv_b, v, nullptr, u, nullptr, B, T, R, true, status, s);
  if (e == cudaSuccess)
    e = launch_gemm_coeffs_bf16(u, params->W_a, params->b_a, params->W_x, params->b_x, params->Lambda, z, ntok, R,
                                status, s);
  if (e == cudaSuccess) {
    // the scan's memset must not clear a status bit the GEMMs above may have set:
    // zero only the ticket and flags here.
    e = cudaMemsetAsync(bytes(workspace) + 4, 0, L.scan.zero_bytes - 4, s);
    if (e == cudaSuccess) {
      ScanArgs a{};
      a.z = z; a.h0 = h0; a.g = g; a.y = pbuf; a.hT = h_T;  // coefficients: no x or conv parameters
      a.status = status;
      a.ticket = reinterpret_cast<unsigned*>(bytes(workspace) + 4);
      a.carry_incl = reinterpret_cast<uint32_t*>(bytes(workspace) + L.scan.off_incl);
      a.carry_agg = reinterpret_cast<uint64_t*>(bytes(workspace) + L.scan.off_agg);
      a.B = B; a.T = T; a.R = R; a.n_cblk = L.scan.n_cblk; a.n_chunks = L.scan.n_chunks;
      a.n_tiles = (int)L.scan.n_tiles; a.pitch = gate_pitch(R);
      e = launch_scan(a, true, s, true);
    }
  }
  if (e == cudaSuccess) e = launch_gemm_bf16(pbuf, W_o, out, ntok, D, R, D, status, s);  // out = p W_oᵀ
  return e;
}

// Queues the scan; with zero_first, first zeroes the status word, the ticket counter and
// the look-back flags (which must be zero when the scan starts).
// coef: z holds the recurrence coefficients of launch_gemm_coeffs_bf16, not pre-activations;
// x, state0 and p are then not read (p may be null).
cudaError_t run_scan(const rglru_params* p, const void* x, const void* z, int64_t pitch, const void* state0,
                     const float* h0, const void* g, void* y, float* hT, int B, int T, int R, bool bf16,
                     const ScanLayout& sl, void* ws, bool zero_first, cudaStream_t s, bool coef = false) {
  if (zero_first) {
    cudaError_t e = cudaMemsetAsync(ws, 0, sl.zero_bytes, s);
    if (e != cudaSuccess) return e;
  }
  ScanArgs a{};
  a.x = x;
  a.z = z;
  a.state0 = state0;
  a.h0 = h0;
  a.g = g;
  a.y = y;
  a.hT = hT;
  if (p != nullptr) {
    a.conv_w = p->conv_w;
    a.conv_b = p->conv_b;
    a.Lambda = p->Lambda;
  }
  a.status = reinterpret_cast<unsigned*>(ws);
  a.ticket = reinterpret_cast<unsigned*>(bytes(ws) + 4);
  a.carry_incl = reinterpret_cast<uint32_t*>(bytes(ws) + sl.off_incl);
  a.carry_agg = reinterpret_cast<uint64_t*>(bytes(ws) + sl.off_agg);
  a.B = B;
  a.T = T;
  a.R = R;
  a.n_cblk = sl.n_cblk;
  a.n_chunks = sl.n_chunks;
  a.n_tiles = (int)sl.n_tiles;
  a.pitch = pitch;
  return launch_scan(a, bf16, s, coef);
}

// ---- fixed scratch of rglru_scan_noalloc ---------------------------------------------
// For callers that cannot allocate device memory, the scan's scratch (status word, tile
// ticket, published chunk states and chunk maps: the layout scan_layout gives, a 256-byte
// header and 12·CW bytes per tile with CW = 128 channels for bf16 and 64 for float32) lives
// in this file-scope array, which
// every GPU that loads the library holds until the process exits. Its name in host code
// is a host-side stand-in, not a device address: the address is looked up once per
// device, with that device current, and handed to the kernels.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

int noalloc_scratch(void** out) {
  static void* addr[kMaxDevices] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e);
  if (dev < 0 || dev >= kMaxDevices) return RGLRU_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* a = nullptr;
    e = cudaGetSymbolAddress(&a, g_noalloc_scratch);
    if (e != cudaSuccess) return fail_cuda(e);
    if (a == nullptr) return fail_cuda(cudaErrorInvalidSymbol);
    addr[dev] = a;
  }
  *out = addr[dev];
  return RGLRU_OK;
}

}  // namespace

extern "C" {

const char* rglru_strerror(int status) {
  switch (status) {
    case RGLRU_OK: return "ok";
    case RGLRU_ERR_NULL: return "a required pointer is NULL";
    case RGLRU_ERR_SHAPE: return "invalid shape (B, T >= 1; R, D >= 8 and multiples of 8; sizes in range)";
    case RGLRU_ERR_ALIGN: return "a pointer is not 16-byte aligned (workspace: 256-byte)";
    case RGLRU_ERR_DTYPE: return "io_dtype not supported by this entry point";
    case RGLRU_ERR_WORKSPACE: return "workspace missing or too small";
    case RGLRU_ERR_CUDA: return "a CUDA call failed (see rglru_last_cuda_error)";
    case RGLRU_ERR_TIMEOUT: return "a bounded wait inside a kernel gave up";
    case RGLRU_ERR_DEVICE: return "the current device is not compute capability 10.0 (B200)";
    default: return "unknown status";
  }
}

int rglru_last_cuda_error(void) { return g_last_cuda_error; }

int rglru_debug_scan_stall(int64_t tile) {
  set_scan_stall(tile < 0 ? -1 : tile);
  return RGLRU_OK;
}
int rglru_version(void) { return 10000; }

int64_t rglru_gate_pitch(int R) { return valid_R(R) ? gate_pitch(R) : 0; }

size_t rglru_scan_workspace_bytes(int B, int T, int R, int io_dtype) {
  if (!valid_dtype(io_dtype) || !valid_R(R) || !valid_tokens(B, T)) return 0;
  return scan_layout(B, T, R, io_dtype == RGLRU_BF16).bytes;
}

size_t rglru_forward_workspace_bytes(int B, int T, int R, int io_dtype) {
  if (!valid_dtype(io_dtype) || !valid_R(R) || !valid_tokens(B, T)) return 0;
  return fwd_layout(B, T, R, io_dtype).bytes;
}

size_t rglru_gate_scan_workspace_bytes(int B, int T, int R, int io_dtype) {
  if (!valid_R(R) || !valid_tokens(B, T) || !fused_ok(io_dtype, T)) return 0;
  return fused_layout(B, T, R).zero_bytes;
}

int rglru_gate_scan(const rglru_params* params, const void* u, const float* h0, void* y, float* h_T, int B, int T,
                    int R, int io_dtype, void* workspace, size_t workspace_bytes, rglru_stream_t stream) {
  const Range range("rglru_gate_scan");
  if (io_dtype != RGLRU_BF16) return RGLRU_ERR_DTYPE;
  if (!valid_R(R) || !valid_tokens(B, T) || T % 128 != 0) return RGLRU_ERR_SHAPE;
  int st = check_params(params);
  if (st != RGLRU_OK) return st;
  if (u == nullptr || y == nullptr) return RGLRU_ERR_NULL;
  if (!aligned16(u) || !aligned16(y) || !aligned16(h0) || !aligned16(h_T)) return RGLRU_ERR_ALIGN;
  const FusedLayout L = fused_layout(B, T, R);
  if (workspace == nullptr || workspace_bytes < L.zero_bytes) return RGLRU_ERR_WORKSPACE;
  if (!aligned256(workspace)) return RGLRU_ERR_ALIGN;
  if ((st = check_device()) != RGLRU_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(workspace, 0, L.zero_bytes, s);
  if (e == cudaSuccess)
    e = launch_gate_scan_bf16(fused_args(params, u, h0, y, h_T, B, T, R, L, workspace), s);
  return e == cudaSuccess ? RGLRU_OK : fail_cuda(e);
}

size_t rglru_step_workspace_bytes(int B, int R, int io_dtype) {
  if (io_dtype != RGLRU_BF16 || !valid_R(R) || !valid_tokens(B, 1)) return 0;
  return step_layout(B, R).bytes;
}

size_t rglru_block_workspace_bytes(int B, int T, int D, int R, int io_dtype) {
  if (io_dtype != RGLRU_BF16 || !valid_R(R) || !valid_R(D) || !valid_tokens(B, T)) return 0;
  return block_layout(B, T, R).bytes;
}

int rglru_conv1d(const float* conv_w, const float* conv_b, const void* x, const void* conv_state0, void* u,
                 void* conv_state_T, int B, int T, int R, int io_dtype, rglru_stream_t stream) {
  const Range range("rglru_conv1d");
  if (!valid_dtype(io_dtype)) return RGLRU_ERR_DTYPE;
  if (!valid_R(R) || !valid_tokens(B, T)) return RGLRU_ERR_SHAPE;
  if (conv_w == nullptr || conv_b == nullptr || x == nullptr || u == nullptr) return RGLRU_ERR_NULL;
  if (!aligned16(conv_w) || !aligned16(conv_b) || !aligned16(x) || !aligned16(u) || !aligned16(conv_state0) ||
      !aligned16(conv_state_T))
    return RGLRU_ERR_ALIGN;
  int st = check_device();
  if (st != RGLRU_OK) return st;
  unsigned* status = global_status_word();
  if (status == nullptr) return fail_cuda(cudaGetLastError());
  cudaError_t e = launch_conv1d(conv_w, conv_b, x, conv_state0, u, conv_state_T, B, T, R, io_dtype == RGLRU_BF16,
                                status, (cudaStream_t)stream);
  return e == cudaSuccess ? RGLRU_OK : fail_cuda(e);
}

int rglru_gate_proj(const void* u, const void* W_a, const float* b_a, const void* W_x, const float* b_x, void* z,
                    int64_t N_tok, int R, int io_dtype, rglru_stream_t stream) {
  const Range range("rglru_gate_proj");
  if (!valid_dtype(io_dtype)) return RGLRU_ERR_DTYPE;
  if (!valid_R(R) || N_tok < 1 || N_tok > (int64_t)INT32_MAX) return RGLRU_ERR_SHAPE;
  if (u == nullptr || W_a == nullptr || b_a == nullptr || W_x == nullptr || b_x == nullptr || z == nullptr)
    return RGLRU_ERR_NULL;
  if (!aligned16(u) || !aligned16(W_a) || !aligned16(b_a) || !aligned16(W_x) || !aligned16(b_x) || !aligned16(z))
    return RGLRU_ERR_ALIGN;
  int st = check_device();
  if (st != RGLRU_OK) return st;
  cudaError_t e;
  if (io_dtype == RGLRU_BF16) {
    unsigned* status = global_status_word();
    if (status == nullptr) return fail_cuda(cudaGetLastError());
    e = launch_gemm_gates_bf16(u, W_a, b_a, W_x, b_x, z, N_tok, R, status, (cudaStream_t)stream);
  } else {
    e = launch_gemm_gates_f32(static_cast<const float*>(u), static_cast<const float*>(W_a), b_a,
                              static_cast<const float*>(W_x), b_x, static_cast<float*>(z), N_tok, R,
                              (cudaStream_t)stream);
  }
  return e == cudaSuccess ? RGLRU_OK : fail_cuda(e);
}

int rglru_scan(const rglru_params* params, const void* x, const void* z, const void* conv_state0, const float* h0,
               const void* gate_g, void* y, float* h_T, int B, int T, int R, int io_dtype, void* workspace,
               size_t workspace_bytes, rglru_stream_t stream) {
  const Range range("rglru_scan");
  if (!valid_dtype(io_dtype)) return RGLRU_ERR_DTYPE;
  if (!valid_R(R) || !valid_tokens(B, T)) return RGLRU_ERR_SHAPE;
  int st = check_params(params);
  if (st != RGLRU_OK) return st;
  if (x == nullptr || z == nullptr || y == nullptr) return RGLRU_ERR_NULL;
  if (!aligned16(x) || !aligned16(z) || !aligned16(y) || !aligned16(conv_state0) || !aligned16(h0) ||
      !aligned16(gate_g) || !aligned16(h_T))
    return RGLRU_ERR_ALIGN;
  const ScanLayout sl = scan_layout(B, T, R, io_dtype == RGLRU_BF16);
  if (workspace == nullptr || workspace_bytes < sl.bytes) return RGLRU_ERR_WORKSPACE;
  if (!aligned256(workspace)) return RGLRU_ERR_ALIGN;
  if ((st = check_device()) != RGLRU_OK) return st;
  cudaError_t e = run_scan(params, x, z, gate_pitch(R), conv_state0, h0, gate_g, y, h_T, B, T, R,
                           io_dtype == RGLRU_BF16, sl, workspace, true, (cudaStream_t)stream);
  return e == cudaSuccess ? RGLRU_OK : fail_cuda(e);
}

int rglru_gate_coeffs(const rglru_params* params, const void* u, void* g, int64_t N_tok, int R,
                      rglru_stream_t stream) {
  const Range range("rglru_gate_coeffs");
  if (!valid_R(R) || N_tok < 1 || N_tok > (int64_t)INT32_MAX) return RGLRU_ERR_SHAPE;
  int st = check_params(params);
  if (st != RGLRU_OK) return st;
  if (u == nullptr || g == nullptr) return RGLRU_ERR_NULL;
  if (!aligned16(u) || !aligned16(g)) return RGLRU_ERR_ALIGN;
  if ((st = check_device()) != RGLRU_OK) return st;
  unsigned* status = global_status_word();
  if (status == nullptr) return fail_cuda(cudaGetLastError());
  cudaError_t e = launch_gemm_coeffs_bf16(u, params->W_a, params->b_a, params->W_x, params->b_x, params->Lambda, g,
                                          N_tok, R, status, (cudaStream_t)stream);
  return e == cudaSuccess ? RGLRU_OK : fail_cuda(e);
}

int rglru_scan_coeffs(const void* g, const float* h0, const void* gate_g, void* y, float* h_T, int B, int T, int R,
                      void* workspace, size_t workspace_bytes, rglru_stream_t stream) {
  const Range range("rglru_scan_coeffs");
  if (!valid_R(R) || !valid_tokens(B, T)) return RGLRU_ERR_SHAPE;
  if (g == nullptr || y == nullptr) return RGLRU_ERR_NULL;
  if (!aligned16(g) || !aligned16(y) || !aligned16(h0) || !aligned16(gate_g) || !aligned16(h_T))
    return RGLRU_ERR_ALIGN;
  const ScanLayout sl = scan_layout(B, T, R, true);
  if (workspace == nullptr || workspace_bytes < sl.bytes) return RGLRU_ERR_WORKSPACE;
  if (!aligned256(workspace)) return RGLRU_ERR_ALIGN;
  int st = check_device();
  if (st != RGLRU_OK) return st;
  cudaError_t e = run_scan(nullptr, nullptr, g, gate_pitch(R), nullptr, h0, gate_g, y, h_T, B, T, R, true, sl,
                           workspace, true, (cudaStream_t)stream, true);
  return e == cudaSuccess ? RGLRU_OK : fail_cuda(e);
}

namespace {
int forward_impl(const rglru_params* params, const void* x, const float* h0, const void* conv_state0, void* y,
                 float* h_T, void* conv_state_T, void* saved, int B, int T, int R, int io_dtype, void* workspace,
                 size_t workspace_bytes, rglru_stream_t stream) {
  if (!valid_dtype(io_dtype)) return RGLRU_ERR_DTYPE;
  if (!valid_R(R) || !valid_tokens(B, T)) return RGLRU_ERR_SHAPE;
  int st = check_params(params);
  if (st != RGLRU_OK) return st;
  if (x == nullptr || y == nullptr) return RGLRU_ERR_NULL;
  if (!aligned16(x) || !aligned16(y) || !aligned16(h0) || !aligned16(conv_state0) || !aligned16(h_T) ||
      !aligned16(conv_state_T))
    return RGLRU_ERR_ALIGN;
  const FwdLayout L = fwd_layout(B, T, R, io_dtype);
  if (workspace == nullptr || workspace_bytes < L.bytes) return RGLRU_ERR_WORKSPACE;
  if (!aligned256(workspace)) return RGLRU_ERR_ALIGN;
  if ((st = check_device()) != RGLRU_OK) return st;
  const bool bf16 = io_dtype == RGLRU_BF16;
  cudaStream_t s = (cudaStream_t)stream;
  void* u = bytes(workspace) + L.off_u;
  void* z = bytes(workspace) + L.off_z;
  unsigned* status = reinterpret_cast<unsigned*>(workspace);
  if (saved == nullptr && fused_faster(io_dtype, T, R)) {
    // the fused path: its chunk carries sit at the start of the workspace (inside the scan's
    // region, which is larger), zeroed with the status word by the conv kernel
    const FusedLayout F = fused_layout(B, T, R);
    if (F.zero_bytes > L.off_u) return RGLRU_ERR_WORKSPACE;  // (never: the scan's region is larger)
    cudaError_t e = launch_conv1d(params->conv_w, params->conv_b, x, conv_state0, u, conv_state_T, B, T, R, true,
                                  status, s, workspace, F.zero_bytes);
    if (e == cudaSuccess) e = launch_gate_scan_bf16(fused_args(params, u, h0, y, h_T, B, T, R, F, workspace), s);
    return e == cudaSuccess ? RGLRU_OK : fail_cuda(e);
  }
  // the conv kernel also zeroes the status word, the scan's ticket and its chunk carries,
  // so that a status bit set by the GEMM or the scan survives until the caller reads it;
  // the GEMM and the scan are launched as programmatic dependents of the kernel before
  cudaError_t e = launch_conv1d(params->conv_w, params->conv_b, x, conv_state0, u, conv_state_T, B, T, R, bf16, status,
                                s, workspace, L.scan.zero_bytes);
  if (e != cudaSuccess) return fail_cuda(e);
  // bf16: the gate GEMM's epilogue forms the recurrence coefficients (d, b) directly
  if (bf16)
    e = launch_gemm_coeffs_bf16(u, params->W_a, params->b_a, params->W_x, params->b_x, params->Lambda, z,
                                (int64_t)B * T, R, status, s, saved);
  else
    e = launch_gemm_gates_f32(static_cast<const float*>(u), static_cast<const float*>(params->W_a), params->b_a,
                              static_cast<const float*>(params->W_x), params->b_x, static_cast<float*>(z),
                              (int64_t)B * T, R, s);
  if (e != cudaSuccess) return fail_cuda(e);
  e = run_scan(params, x, z, gate_pitch(R), conv_state0, h0, nullptr, y, h_T, B, T, R, bf16, L.scan, workspace,
               false, s, bf16);
  return e == cudaSuccess ? RGLRU_OK : fail_cuda(e);
}
}  // namespace

int rglru_forward(const rglru_params* params, const void* x, const float* h0, const void* conv_state0, void* y,
                  float* h_T, void* conv_state_T, int B, int T, int R, int io_dtype, void* workspace,
                  size_t workspace_bytes, rglru_stream_t stream) {
  const Range range("rglru_forward");
  return forward_impl(params, x, h0, conv_state0, y, h_T, conv_state_T, nullptr, B, T, R, io_dtype, workspace,
                      workspace_bytes, stream);
}

int rglru_forward_kernels(int B, int T, int R, int io_dtype) {
  if (!valid_dtype(io_dtype) || !valid_R(R) || !valid_tokens(B, T)) return 0;
  return fused_faster(io_dtype, T, R) ? 2 : 3;
}

size_t rglru_saved_bytes(int B, int T, int R) {
  if (!valid_R(R) || !valid_tokens(B, T)) return 0;
  return (size_t)B * T * gate_pitch(R) * 2;
}

int rglru_forward_train(const rglru_params* params, const void* x, const float* h0, const void* conv_state0, void* y,
                        float* h_T, void* conv_state_T, void* saved, int B, int T, int R, void* workspace,
                        size_t workspace_bytes, rglru_stream_t stream) {
  const Range range("rglru_forward_train");
  if (saved == nullptr) return RGLRU_ERR_NULL;
  if (!aligned16(saved)) return RGLRU_ERR_ALIGN;
  return forward_impl(params, x, h0, conv_state0, y, h_T, conv_state_T, saved, B, T, R, RGLRU_BF16, workspace,
                      workspace_bytes, stream);
}

int rglru_step(const rglru_params* params, const void* x_t, void* conv_state, float* h, void* y_t, int B, int R,
               int64_t step, int io_dtype, void* workspace, size_t workspace_bytes, rglru_stream_t stream) {
  const Range range("rglru_step");
  if (io_dtype != RGLRU_BF16) return RGLRU_ERR_DTYPE;
  if (!valid_R(R) || !valid_tokens(B, 1) || step < 0) return RGLRU_ERR_SHAPE;
  int st = check_params(params);
  if (st != RGLRU_OK) return st;
  if (x_t == nullptr || conv_state == nullptr || h == nullptr || y_t == nullptr) return RGLRU_ERR_NULL;
  if (!aligned16(x_t) || !aligned16(conv_state) || !aligned16(h) || !aligned16(y_t)) return RGLRU_ERR_ALIGN;
  const StepLayout L = step_layout(B, R);
  if (workspace == nullptr || workspace_bytes < L.bytes) return RGLRU_ERR_WORKSPACE;
  if (!aligned256(workspace)) return RGLRU_ERR_ALIGN;
  if ((st = check_device()) != RGLRU_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  float* cla = reinterpret_cast<float*>(bytes(workspace) + L.off_cla);
  void* u_t = bytes(workspace) + L.off_u;
  float* u_f32 = reinterpret_cast<float*>(bytes(workspace) + L.off_uf);
  unsigned* status = reinterpret_cast<unsigned*>(workspace);
  cudaError_t e = launch_decode_conv(params->conv_w, params->conv_b, params->Lambda, x_t, conv_state, step, u_t,
                                     u_f32, cla, status, B, R, s);
  if (e != cudaSuccess) return fail_cuda(e);
  e = launch_gemm_step_bf16(u_t, u_f32, params->W_a, params->b_a, params->W_x, params->b_x, cla, h, y_t, B, R,
                            status, s);
  return e == cudaSuccess ? RGLRU_OK : fail_cuda(e);
}

int rglru_gemm_bf16(const void* A, const void* Bm, void* C, int64_t M, int N, int K, rglru_stream_t stream) {
  const Range range("rglru_gemm_bf16");
  if (M < 1 || M > (int64_t)INT32_MAX * 128 || !valid_R(N) || !valid_R(K)) return RGLRU_ERR_SHAPE;
  if (A == nullptr || Bm == nullptr || C == nullptr) return RGLRU_ERR_NULL;
  if (!aligned16(A) || !aligned16(Bm) || !aligned16(C)) return RGLRU_ERR_ALIGN;
  int st = check_device();
  if (st != RGLRU_OK) return st;
  unsigned* status = global_status_word();
  if (status == nullptr) return fail_cuda(cudaGetLastError());
  cudaError_t e = launch_gemm_bf16(A, Bm, C, M, N, K, N, status, (cudaStream_t)stream);
  return e == cudaSuccess ? RGLRU_OK : fail_cuda(e);
}

size_t rglru_backward_workspace_bytes(int B, int T, int R) {
  if (!valid_R(R) || !valid_tokens(B, T)) return 0;
  return bwd_layout(B, T, R).bytes;
}

namespace {
int backward_impl(const rglru_params* params, const void* x, const void* y, const void* dy, const float* h0,
                  const float* dh_T, const void* conv_state0, const void* saved, const rglru_grads* grads, int B,
                  int T, int R, void* workspace, size_t workspace_bytes, rglru_stream_t stream) {
  if (!valid_R(R) || !valid_tokens(B, T)) return RGLRU_ERR_SHAPE;
  // the chunked kernels index (batch row, 64-step chunk) with the grid's y dimension
  if ((int64_t)B * ((T + kScanTC - 1) / kScanTC) > 65535) return RGLRU_ERR_SHAPE;
  int st = check_params(params);
  if (st != RGLRU_OK) return st;
  if (x == nullptr || y == nullptr || dy == nullptr || grads == nullptr) return RGLRU_ERR_NULL;
  if (!aligned16(saved)) return RGLRU_ERR_ALIGN;
  const rglru_grads& g = *grads;
  if (g.dx == nullptr || g.dconv_w == nullptr || g.dconv_b == nullptr || g.dW_a == nullptr || g.db_a == nullptr ||
      g.dW_x == nullptr || g.db_x == nullptr || g.dLambda == nullptr)
    return RGLRU_ERR_NULL;
  if (!aligned16(x) || !aligned16(y) || !aligned16(dy) || !aligned16(h0) || !aligned16(dh_T) ||
      !aligned16(conv_state0) || !aligned16(g.dx) || !aligned16(g.dconv_state0) || !aligned16(g.dconv_w) ||
      !aligned16(g.dconv_b) || !aligned16(g.dW_a) || !aligned16(g.db_a) || !aligned16(g.dW_x) ||
      !aligned16(g.db_x) || !aligned16(g.dLambda) || !aligned16(g.dh0))
    return RGLRU_ERR_ALIGN;
  const BwdLayout L = bwd_layout(B, T, R);
  if (workspace == nullptr || workspace_bytes < L.bytes) return RGLRU_ERR_WORKSPACE;
  if (!aligned256(workspace)) return RGLRU_ERR_ALIGN;
  if ((st = check_device()) != RGLRU_OK) return st;
  BwdArgs a{};
  a.x = x; a.y = y; a.dy = dy; a.h0 = h0; a.dh_T = dh_T; a.state0 = conv_state0;
  a.conv_w = params->conv_w; a.conv_b = params->conv_b; a.W_a = params->W_a; a.b_a = params->b_a;
  a.W_x = params->W_x; a.b_x = params->b_x; a.Lambda = params->Lambda;
  a.dx = g.dx; a.dstate0 = g.dconv_state0; a.dconv_w = g.dconv_w; a.dconv_b = g.dconv_b; a.dW_a = g.dW_a;
  a.db_a = g.db_a; a.dW_x = g.dW_x; a.db_x = g.db_x; a.dLambda = g.dLambda; a.dh0 = g.dh0;
  a.z_saved = saved;
  a.B = B; a.T = T; a.R = R;
  cudaError_t e = launch_backward(a, L, workspace, (cudaStream_t)stream);
  return e == cudaSuccess ? RGLRU_OK : fail_cuda(e);
}
}  // namespace

int rglru_backward(const rglru_params* params, const void* x, const void* y, const void* dy, const float* h0,
                   const float* dh_T, const void* conv_state0, const rglru_grads* grads, int B, int T, int R,
                   void* workspace, size_t workspace_bytes, rglru_stream_t stream) {
  const Range range("rglru_backward");
  return backward_impl(params, x, y, dy, h0, dh_T, conv_state0, nullptr, grads, B, T, R, workspace, workspace_bytes,
                       stream);
}

int rglru_backward_saved(const rglru_params* params, const void* x, const void* y, const void* dy, const float* h0,
                         const float* dh_T, const void* conv_state0, const void* saved, const rglru_grads* grads,
                         int B, int T, int R, void* workspace, size_t workspace_bytes, rglru_stream_t stream) {
  const Range range("rglru_backward_saved");
  if (saved == nullptr) return RGLRU_ERR_NULL;
  return backward_impl(params, x, y, dy, h0, dh_T, conv_state0, saved, grads, B, T, R, workspace, workspace_bytes,
                       stream);
}

int rglru_block_forward(const rglru_params* params, const void* W_1, const void* W_2, const void* W_o, const void* x,
                        const float* h0, void* out, float* h_T, int B, int T, int D, int R, int io_dtype,
                        void* workspace, size_t workspace_bytes, rglru_stream_t stream) {
  const Range range("rglru_block_forward");
  if (io_dtype != RGLRU_BF16) return RGLRU_ERR_DTYPE;
  if (!valid_R(R) || !valid_R(D) || !valid_tokens(B, T)) return RGLRU_ERR_SHAPE;
  int st = check_params(params);
  if (st != RGLRU_OK) return st;
  if (W_1 == nullptr || W_2 == nullptr || W_o == nullptr || x == nullptr || out == nullptr) return RGLRU_ERR_NULL;
  if (!aligned16(W_1) || !aligned16(W_2) || !aligned16(W_o) || !aligned16(x) || !aligned16(out) ||
      !aligned16(h0) || !aligned16(h_T))
    return RGLRU_ERR_ALIGN;
  const BlockLayout L = block_layout(B, T, R);
  if (workspace == nullptr || workspace_bytes < L.bytes) return RGLRU_ERR_WORKSPACE;
  if (!aligned256(workspace)) return RGLRU_ERR_ALIGN;
  if ((st = check_device()) != RGLRU_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(workspace, 0, 4, s);
  if (e == cudaSuccess) e = block_sequence(params, W_1, W_2, W_o, x, h0, out, h_T, B, T, D, R, L, workspace, s);
  return e == cudaSuccess ? RGLRU_OK : fail_cuda(e);
}

size_t rglru_layer_workspace_bytes(int B, int T, int D, int R, int H, int io_dtype) {
  if (io_dtype != RGLRU_BF16 || !valid_R(R) || !valid_R(D) || !valid_R(H) || !valid_tokens(B, T)) return 0;
  return layer_layout(B, T, D, R, H).bytes;
}

int rglru_layer_forward(const rglru_params* params, const rglru_layer_weights* w, const void* x, const float* h0,
                        void* out, float* h_T, int B, int T, int D, int R, int H, float eps, int io_dtype,
                        void* workspace, size_t workspace_bytes, rglru_stream_t stream) {
  const Range range("rglru_layer_forward");
  if (io_dtype != RGLRU_BF16) return RGLRU_ERR_DTYPE;
  if (!valid_R(R) || !valid_R(D) || !valid_R(H) || !valid_tokens(B, T)) return RGLRU_ERR_SHAPE;
  if (!(eps >= 0.0f) || eps > 1.0f) return RGLRU_ERR_SHAPE;  // also rejects NaN
  int st = check_params(params);
  if (st != RGLRU_OK) return st;
  if (w == nullptr || x == nullptr || out == nullptr) return RGLRU_ERR_NULL;
  if (w->norm1_scale == nullptr || w->W_1 == nullptr || w->W_2 == nullptr || w->W_o == nullptr ||
      w->norm2_scale == nullptr || w->W_gate == nullptr || w->W_up == nullptr || w->W_down == nullptr)
    return RGLRU_ERR_NULL;
  if (!aligned16(w->norm1_scale) || !aligned16(w->W_1) || !aligned16(w->W_2) || !aligned16(w->W_o) ||
      !aligned16(w->norm2_scale) || !aligned16(w->W_gate) || !aligned16(w->W_up) || !aligned16(w->W_down) ||
      !aligned16(x) || !aligned16(out) || !aligned16(h0) || !aligned16(h_T))
    return RGLRU_ERR_ALIGN;
  if (out == x) return RGLRU_ERR_SHAPE;  // the residual stream is read after out is written
  const LayerLayout L = layer_layout(B, T, D, R, H);
  if (workspace == nullptr || workspace_bytes < L.bytes) return RGLRU_ERR_WORKSPACE;
  if (!aligned256(workspace)) return RGLRU_ERR_ALIGN;
  if ((st = check_device()) != RGLRU_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const int64_t ntok = (int64_t)B * T;
  void* nrm = bytes(workspace) + L.off_n;
  void* o = bytes(workspace) + L.off_o;
  void* yres = bytes(workspace) + L.off_y;
  void* gate = bytes(workspace) + L.off_gate;
  void* up = bytes(workspace) + L.off_up;
  unsigned* status = reinterpret_cast<unsigned*>(workspace);
  cudaError_t e = cudaMemsetAsync(workspace, 0, 4, s);
  // y = x + RecurrentBlock(RMSNorm₁(x))
  if (e == cudaSuccess) e = launch_add_rmsnorm(x, nullptr, nullptr, nrm, w->norm1_scale, ntok, D, eps, s);
  if (e == cudaSuccess)
    e = block_sequence(params, w->W_1, w->W_2, w->W_o, nrm, h0, o, h_T, B, T, D, R, L.block, workspace, s);
  if (e == cudaSuccess) e = launch_add_rmsnorm(x, o, yres, nrm, w->norm2_scale, ntok, D, eps, s);
  // out = y + (GeLU(n W_gateᵀ) ⊙ n W_upᵀ) W_downᵀ
  if (e == cudaSuccess) e = launch_gemm_bf16(nrm, w->W_gate, gate, ntok, H, D, H, status, s);
  if (e == cudaSuccess) e = launch_gemm_bf16(nrm, w->W_up, up, ntok, H, D, H, status, s);
  if (e == cudaSuccess) e = launch_gelu_mul(gate, up, gate, ntok * H, s);
  if (e == cudaSuccess) e = launch_gemm_bf16(gate, w->W_down, o, ntok, D, H, D, status, s);
  if (e == cudaSuccess) e = launch_add_rmsnorm(yres, o, out, nullptr, nullptr, ntok, D, eps, s);
  return e == cudaSuccess ? RGLRU_OK : fail_cuda(e);
}

size_t rglru_layer_step_workspace_bytes(int B, int D, int R, int H, int io_dtype) {
  if (io_dtype != RGLRU_BF16 || !valid_R(R) || !valid_R(D) || !valid_R(H) || !valid_tokens(B, 1)) return 0;
  return layer_step_layout(B, D, R, H).bytes;
}

int rglru_layer_step(const rglru_params* params, const rglru_layer_weights* w, const void* x_t, void* conv_state,
                     float* h, void* out_t, int B, int D, int R, int H, int64_t step, float eps, int io_dtype,
                     void* workspace, size_t workspace_bytes, rglru_stream_t stream) {
  const Range range("rglru_layer_step");
  if (io_dtype != RGLRU_BF16) return RGLRU_ERR_DTYPE;
  if (!valid_R(R) || !valid_R(D) || !valid_R(H) || !valid_tokens(B, 1) || step < 0) return RGLRU_ERR_SHAPE;
  if (!(eps >= 0.0f) || eps > 1.0f) return RGLRU_ERR_SHAPE;  // also rejects NaN
  int st = check_params(params);
  if (st != RGLRU_OK) return st;
  if (w == nullptr || x_t == nullptr || conv_state == nullptr || h == nullptr || out_t == nullptr)
    return RGLRU_ERR_NULL;
  if (w->norm1_scale == nullptr || w->W_1 == nullptr || w->W_2 == nullptr || w->W_o == nullptr ||
      w->norm2_scale == nullptr || w->W_gate == nullptr || w->W_up == nullptr || w->W_down == nullptr)
    return RGLRU_ERR_NULL;
  if (!aligned16(w->norm1_scale) || !aligned16(w->W_1) || !aligned16(w->W_2) || !aligned16(w->W_o) ||
      !aligned16(w->norm2_scale) || !aligned16(w->W_gate) || !aligned16(w->W_up) || !aligned16(w->W_down) ||
      !aligned16(x_t) || !aligned16(conv_state) || !aligned16(h) || !aligned16(out_t))
    return RGLRU_ERR_ALIGN;
  if (out_t == x_t) return RGLRU_ERR_SHAPE;  // the residual stream is read after out_t is written
  const LayerStepLayout L = layer_step_layout(B, D, R, H);
  if (workspace == nullptr || workspace_bytes < L.bytes) return RGLRU_ERR_WORKSPACE;
  if (!aligned256(workspace)) return RGLRU_ERR_ALIGN;
  if ((st = check_device()) != RGLRU_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* ws = bytes(workspace);
  unsigned* status = reinterpret_cast<unsigned*>(ws);
  unsigned* conv_word = reinterpret_cast<unsigned*>(ws + 4);  // the decode conv zeroes its word
  float* cla = reinterpret_cast<float*>(ws + L.step.off_cla);
  void* u_t = ws + L.step.off_u;
  float* u_f32 = reinterpret_cast<float*>(ws + L.step.off_uf);
  void* nrm = ws + L.off_n;
  void* v = ws + L.off_v;
  void* g = ws + L.off_g;
  void* y = ws + L.off_y;
  void* o = ws + L.off_o;
  void* res = ws + L.off_res;
  void* gate = ws + L.off_gate;
  void* up = ws + L.off_up;
  cudaError_t e = cudaMemsetAsync(workspace, 0, 4, s);
  // residual stream + RecurrentBlock(RMSNorm₁(x_t)) with one RG-LRU decode step
  if (e == cudaSuccess) e = launch_add_rmsnorm(x_t, nullptr, nullptr, nrm, w->norm1_scale, B, D, eps, s);
  if (e == cudaSuccess) e = launch_gemm_bf16(nrm, w->W_1, v, B, R, D, R, status, s);  // v_t = n W_1ᵀ
  if (e == cudaSuccess) e = launch_gemm_bf16(nrm, w->W_2, g, B, R, D, R, status, s);  // g_t = n W_2ᵀ
  if (e == cudaSuccess)
    e = launch_decode_conv(params->conv_w, params->conv_b, params->Lambda, v, conv_state, step, u_t, u_f32, cla,
                           conv_word, B, R, s);
  if (e == cudaSuccess)
    e = launch_gemm_step_bf16(u_t, u_f32, params->W_a, params->b_a, params->W_x, params->b_x, cla, h, y, B, R,
                              status, s);
  if (e == cudaSuccess) e = launch_gelu_mul(g, y, g, (int64_t)B * R, s);  // h ⊙ GeLU(g_t)
  if (e == cudaSuccess) e = launch_gemm_bf16(g, w->W_o, o, B, D, R, D, status, s);
  if (e == cudaSuccess) e = launch_add_rmsnorm(x_t, o, res, nrm, w->norm2_scale, B, D, eps, s);
  // + MLP(RMSNorm₂(·))
  if (e == cudaSuccess) e = launch_gemm_bf16(nrm, w->W_gate, gate, B, H, D, H, status, s);
  if (e == cudaSuccess) e = launch_gemm_bf16(nrm, w->W_up, up, B, H, D, H, status, s);
  if (e == cudaSuccess) e = launch_gelu_mul(gate, up, gate, (int64_t)B * H, s);
  if (e == cudaSuccess) e = launch_gemm_bf16(gate, w->W_down, o, B, D, H, D, status, s);
  if (e == cudaSuccess) e = launch_add_rmsnorm(res, o, out_t, nullptr, nullptr, B, D, eps, s);
  return e == cudaSuccess ? RGLRU_OK : fail_cuda(e);
}

size_t rglru_attention_step_workspace_bytes(int B, int D, int window) {
  if (!valid_attention(B, D, window)) return 0;
  return attn_layout(B, D, window).bytes;
}

int rglru_attention_step(const rglru_attention_weights* w, const void* x_t, void* k_ring, void* v_ring, void* out_t,
                         int B, int D, int window, int64_t pos, void* workspace, size_t workspace_bytes,
                         rglru_stream_t stream) {
  const Range range("rglru_attention_step");
  if (!valid_attention(B, D, window) || pos < 0) return RGLRU_ERR_SHAPE;
  if (w == nullptr || w->W_qkv == nullptr || w->W_o == nullptr || x_t == nullptr || k_ring == nullptr ||
      v_ring == nullptr || out_t == nullptr)
    return RGLRU_ERR_NULL;
  if (!aligned16(w->W_qkv) || !aligned16(w->W_o) || !aligned16(x_t) || !aligned16(k_ring) || !aligned16(v_ring) ||
      !aligned16(out_t))
    return RGLRU_ERR_ALIGN;
  const AttnLayout L = attn_layout(B, D, window);
  if (workspace == nullptr || workspace_bytes < L.bytes) return RGLRU_ERR_WORKSPACE;
  if (!aligned256(workspace)) return RGLRU_ERR_ALIGN;
  int st = check_device();
  if (st != RGLRU_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(workspace, 0, 4, s);
  if (e == cudaSuccess) e = attention_sequence(w, x_t, k_ring, v_ring, out_t, B, D, window, pos, L, workspace, s);
  return e == cudaSuccess ? RGLRU_OK : fail_cuda(e);
}

size_t rglru_attention_layer_step_workspace_bytes(int B, int D, int H, int window) {
  if (!valid_attention(B, D, window) || !valid_R(H)) return 0;
  return attn_layer_layout(B, D, H, window).bytes;
}

int rglru_attention_layer_step(const rglru_attention_layer_weights* w, const void* x_t, void* k_ring, void* v_ring,
                               void* out_t, int B, int D, int H, int window, int64_t pos, float eps,
                               void* workspace, size_t workspace_bytes, rglru_stream_t stream) {
  const Range range("rglru_attention_layer_step");
  if (!valid_attention(B, D, window) || !valid_R(H) || pos < 0) return RGLRU_ERR_SHAPE;
  if (!(eps >= 0.0f) || eps > 1.0f) return RGLRU_ERR_SHAPE;  // also rejects NaN
  if (w == nullptr || w->norm1_scale == nullptr || w->W_qkv == nullptr || w->W_o == nullptr ||
      w->norm2_scale == nullptr || w->W_gate == nullptr || w->W_up == nullptr || w->W_down == nullptr ||
      x_t == nullptr || k_ring == nullptr || v_ring == nullptr || out_t == nullptr)
    return RGLRU_ERR_NULL;
  if (!aligned16(w->norm1_scale) || !aligned16(w->W_qkv) || !aligned16(w->W_o) || !aligned16(w->norm2_scale) ||
      !aligned16(w->W_gate) || !aligned16(w->W_up) || !aligned16(w->W_down) || !aligned16(x_t) ||
      !aligned16(k_ring) || !aligned16(v_ring) || !aligned16(out_t))
    return RGLRU_ERR_ALIGN;
  if (out_t == x_t) return RGLRU_ERR_SHAPE;  // the residual stream is read after out_t is written
  const AttnLayerLayout L = attn_layer_layout(B, D, H, window);
  if (workspace == nullptr || workspace_bytes < L.bytes) return RGLRU_ERR_WORKSPACE;
  if (!aligned256(workspace)) return RGLRU_ERR_ALIGN;
  int st = check_device();
  if (st != RGLRU_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* ws = bytes(workspace);
  unsigned* status = reinterpret_cast<unsigned*>(ws);
  void* nrm = ws + L.off_n;
  void* o = ws + L.off_o;
  void* res = ws + L.off_res;
  void* gate = ws + L.off_gate;
  void* up = ws + L.off_up;
  const rglru_attention_weights aw{w->W_qkv, w->W_o};
  cudaError_t e = cudaMemsetAsync(workspace, 0, 4, s);
  // residual stream + LocalMQA(RMSNorm₁(x_t))
  if (e == cudaSuccess) e = launch_add_rmsnorm(x_t, nullptr, nullptr, nrm, w->norm1_scale, B, D, eps, s);
  if (e == cudaSuccess) e = attention_sequence(&aw, nrm, k_ring, v_ring, o, B, D, window, pos, L.attn, workspace, s);
  if (e == cudaSuccess) e = launch_add_rmsnorm(x_t, o, res, nrm, w->norm2_scale, B, D, eps, s);
  // + MLP(RMSNorm₂(·))
  if (e == cudaSuccess) e = launch_gemm_bf16(nrm, w->W_gate, gate, B, H, D, H, status, s);
  if (e == cudaSuccess) e = launch_gemm_bf16(nrm, w->W_up, up, B, H, D, H, status, s);
  if (e == cudaSuccess) e = launch_gelu_mul(gate, up, gate, (int64_t)B * H, s);
  if (e == cudaSuccess) e = launch_gemm_bf16(gate, w->W_down, o, B, D, H, D, status, s);
  if (e == cudaSuccess) e = launch_add_rmsnorm(res, o, out_t, nullptr, nullptr, B, D, eps, s);
  return e == cudaSuccess ? RGLRU_OK : fail_cuda(e);
}

int rglru_scan_noalloc(const rglru_params* params, const void* x, const void* z, const void* conv_state0,
                       const float* h0, const void* gate_g, void* y, float* h_T, int B, int T, int R, int io_dtype,
                       rglru_stream_t stream) {
  const Range range("rglru_scan_noalloc");
  if (!valid_dtype(io_dtype)) return RGLRU_ERR_DTYPE;
  if (!valid_R(R) || !valid_tokens(B, T)) return RGLRU_ERR_SHAPE;
  int st = check_params(params);
  if (st != RGLRU_OK) return st;
  if (x == nullptr || z == nullptr || y == nullptr) return RGLRU_ERR_NULL;
  if (!aligned16(x) || !aligned16(z) || !aligned16(y) || !aligned16(conv_state0) || !aligned16(h0) ||
      !aligned16(gate_g) || !aligned16(h_T))
    return RGLRU_ERR_ALIGN;
  const ScanLayout sl = scan_layout(B, T, R, io_dtype == RGLRU_BF16);
  if (sl.bytes > kNoAllocScratchBytes) return RGLRU_ERR_WORKSPACE;  // beyond the fixed scratch
  if ((st = check_device()) != RGLRU_OK) return st;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != RGLRU_OK) return st;
  // the array keeps the previous call's contents: run_scan clears the status word, the
  // ticket and the chunk states this call uses before its kernel starts
  cudaError_t e = run_scan(params, x, z, gate_pitch(R), conv_state0, h0, gate_g, y, h_T, B, T, R,
                           io_dtype == RGLRU_BF16, sl, scratch, true, (cudaStream_t)stream);
  return e == cudaSuccess ? RGLRU_OK : fail_cuda(e);
}

int rglru_scan_noalloc_status(rglru_stream_t stream) {
  const int st = check_device();
  if (st != RGLRU_OK) return st;
  void* scratch = nullptr;
  const int sa = noalloc_scratch(&scratch);
  if (sa != RGLRU_OK) return sa;
  return rglru_workspace_status(scratch, stream);
}

int rglru_workspace_status(void* workspace, rglru_stream_t stream) {
  unsigned* word = workspace != nullptr ? reinterpret_cast<unsigned*>(workspace) : global_status_word();
  if (word == nullptr) return fail_cuda(cudaGetLastError());
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return fail_cuda(e);
  unsigned v = 0;
  e = cudaMemcpy(&v, word, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail_cuda(e);
  e = cudaMemset(word, 0, sizeof(v));
  if (e != cudaSuccess) return fail_cuda(e);
  return (v & kStatusTimeout) ? RGLRU_ERR_TIMEOUT : RGLRU_OK;
}

}  // extern "C"
