// rglru_scan_noalloc: the fused RG-LRU scan for callers that cannot allocate device
// memory.
//
// Who needs this: code that is handed only its input and output buffers and has no way
// to obtain more device memory — for example a custom operator inside a host framework
// that owns the allocator and exposes none to plugins, a serving loop whose memory was
// fully reserved at start-up and must not grow, or a latency-critical path where a
// cudaMalloc could synchronise the device. Such callers cannot provide the scan's
// workspace (its tile ticket, look-back flags and chunk carries).
//
// What it does instead: the scratch lives in one file-scope device array of fixed size,
// kNoAllocScratchBytes, which every GPU that loads this library keeps until the process
// exits. Host code cannot use the array's name as a device address (it only names a
// host-side stand-in), so on the first call on each device the entry point looks up the
// array's device address with cudaGetSymbolAddress, with that device current, and passes
// that address to the kernel. Nothing is allocated or freed, by this code or by any
// library it calls.
#include <cstdint>
#include <cuda_runtime.h>
#include <mutex>

#include "../../include/rglru.h"
#include "kernels.cuh"

using namespace rglru;

namespace {

// 8 MiB per device: enough for B·⌈R/128⌉·⌈T/64⌉ ≈ 5400 bf16 tiles of 128 channels
// (12 bytes of carries per channel; e.g. B=8, T=2048, R=2048 needs 4096 tiles) or
// ≈ 10900 float32 tiles of 64 channels.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDev = 64;
void* g_scratch_addr[kMaxDev] = {nullptr};
std::mutex g_scratch_mu;

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device address of the scratch array on the current device (looked up once per device).
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return RGLRU_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDev) return RGLRU_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) return RGLRU_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return RGLRU_OK;
}

}  // namespace

extern "C" RGLRU_API int rglru_scan_noalloc(const rglru_params* p, const void* x, const void* z,
                                            const void* conv_state0, const float* h0, const void* gate_g, void* y,
                                            float* h_T, int B, int T, int R, int io_dtype, rglru_stream_t stream) {
  if (io_dtype != RGLRU_F32 && io_dtype != RGLRU_BF16) return RGLRU_ERR_DTYPE;
  if (R < 8 || R % 8 != 0 || R > 65536 || B < 1 || T < 1 || B > 65535 || (int64_t)B * T > (int64_t)INT32_MAX)
    return RGLRU_ERR_SHAPE;
  if (p == nullptr || p->conv_w == nullptr || p->conv_b == nullptr || p->Lambda == nullptr || x == nullptr ||
      z == nullptr || y == nullptr)
    return RGLRU_ERR_NULL;
  if (!al16(p->conv_w) || !al16(p->conv_b) || !al16(p->Lambda) || !al16(x) || !al16(z) || !al16(y) ||
      !al16(conv_state0) || !al16(h0) || !al16(gate_g) || !al16(h_T))
    return RGLRU_ERR_ALIGN;
  const bool bf16 = io_dtype == RGLRU_BF16;
  const ScanLayout sl = scan_layout(B, T, R, bf16);
  if (sl.bytes > kNoAllocScratchBytes) return RGLRU_ERR_WORKSPACE;  // problem too large for the fixed scratch
  int dev = 0, major = 0, minor = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (e != cudaSuccess) return RGLRU_ERR_CUDA;
  if (major * 10 + minor != 100) return RGLRU_ERR_DEVICE;

  void* scratch = nullptr;
  int st = scratch_address(&scratch);
  if (st != RGLRU_OK) return st;
  unsigned* status = global_status_word();
  if (status == nullptr) return RGLRU_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  // The array keeps whatever the previous call left in it: the ticket counter and the
  // published carries must start at zero, so the used part is cleared first.
  e = cudaMemsetAsync(scratch, 0, sl.zero_bytes, s);
  if (e != cudaSuccess) return RGLRU_ERR_CUDA;
  ScanArgs a{};
  a.x = x;
  a.z = z;
  a.state0 = conv_state0;
  a.h0 = h0;
  a.g = gate_g;
  a.y = y;
  a.hT = h_T;
  a.conv_w = p->conv_w;
  a.conv_b = p->conv_b;
  a.Lambda = p->Lambda;
  a.status = status;
  a.ticket = reinterpret_cast<unsigned*>(static_cast<unsigned char*>(scratch) + 4);
  a.carry_incl = reinterpret_cast<uint32_t*>(static_cast<unsigned char*>(scratch) + sl.off_incl);
  a.B = B;
  a.T = T;
  a.R = R;
  a.n_cblk = sl.n_cblk;
  a.n_chunks = sl.n_chunks;
  a.n_tiles = (int)sl.n_tiles;
  a.pitch = gate_pitch(R);
  e = launch_scan(a, bf16, s);
  if (e != cudaSuccess) return RGLRU_ERR_CUDA;
  return RGLRU_OK;
}
