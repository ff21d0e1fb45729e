// fs_lm_head_argmax_noalloc: the final RMSNorm + tied LM head + greedy
// selection for callers that must not allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is off limits — a host
// thread with a latency budget (cudaMalloc can block on a device-wide
// synchronisation and take driver locks), a process whose device memory is
// entirely reserved by another framework's pool, or an embedding that hands
// us buffers and forbids us to own any. Such a caller passes its inputs and
// outputs; the two scratch areas this computation needs (the normalised rows
// and the per-block argmax partials) live in one fixed array compiled into
// the library instead of coming from cudaMalloc.
#include <mutex>
#include <string>

#include "runtime.h"

namespace {

// Size of the fixed scratch array. Every GPU that loads libfs holds it
// until the process exits.
constexpr size_t kNoAllocScratchBytes = 512u << 10;  // 512 KiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool on_device(const void* p) {
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged;
}

}  // namespace

extern "C" fs_status fs_lm_head_argmax_noalloc(const void* embed, const void* final_norm,
                                               int32_t hidden, int32_t vocab, float rms_eps,
                                               const float* x, int32_t rows, float* logits,
                                               int32_t* argmax, void* stream) {
  using fs::set_error;
  if (!embed || !final_norm || !x || (!logits && !argmax)) {
    set_error("fs_lm_head_argmax_noalloc: embed, final_norm, x and one output are required");
    return FS_ERR_NULL;
  }
  if (hidden <= 0 || hidden % 64 || vocab <= 0 || rows <= 0 || rows > fs::kMaxBatch ||
      !(rms_eps > 0.f)) {
    set_error("fs_lm_head_argmax_noalloc: need hidden % 64 == 0, vocab > 0, 1 <= rows <= 64, "
              "rms_eps > 0");
    return FS_ERR_INVALID;
  }
  if (!aligned(embed, 16) || !aligned(final_norm, 16) || !aligned(x, 16) ||
      (logits && !aligned(logits, 16)) || (argmax && !aligned(argmax, 4))) {
    set_error("fs_lm_head_argmax_noalloc: misaligned pointer");
    return FS_ERR_ALIGN;
  }
  if (!on_device(embed) || !on_device(final_norm) || !on_device(x) ||
      (logits && !on_device(logits)) || (argmax && !on_device(argmax))) {
    set_error("fs_lm_head_argmax_noalloc: every pointer must be device memory");
    return FS_ERR_INVALID;
  }
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    set_error("fs_lm_head_argmax_noalloc: cannot query the current device");
    return FS_ERR_CUDA;
  }
  const int n_part = 4 * sms;
  // Scratch layout: normalised rows fp32 [rows, hidden], then the argmax
  // partials float2 [rows, n_part]. Both are fully written before they are
  // read, so nothing in the array has to start at zero.
  const size_t xf_bytes = round_up((size_t)rows * hidden * sizeof(float), 256);
  const size_t part_bytes = (size_t)rows * n_part * sizeof(float2);
  if (xf_bytes + part_bytes > kNoAllocScratchBytes) {
    set_error("fs_lm_head_argmax_noalloc: rows * hidden * 4 + rows * " + std::to_string(n_part) +
              " * 8 bytes exceeds the fixed 512 KiB scratch array");
    return FS_ERR_INVALID;
  }
  void* base = nullptr;
  {
    // The array's device address: looked up again on every call made outside
    // a stream capture (so a context torn down by cudaDeviceReset and made
    // anew never leaves a stale address behind), and taken from the last
    // lookup inside a capture, where the lookup is not allowed.
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(static_cast<cudaStream_t>(stream), &cap) != cudaSuccess) {
      cudaGetLastError();
      cap = cudaStreamCaptureStatusNone;
    }
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (cap == cudaStreamCaptureStatusNone) g_noalloc_addr[dev] = nullptr;
    if (!g_noalloc_addr[dev]) {
      cudaError_t e = cudaGetSymbolAddress(&g_noalloc_addr[dev], g_noalloc_scratch);
      if (e != cudaSuccess) {
        g_noalloc_addr[dev] = nullptr;
        set_error(std::string("fs_lm_head_argmax_noalloc: cudaGetSymbolAddress failed: ") +
                  cudaGetErrorString(e));
        return FS_ERR_CUDA;
      }
    }
    base = g_noalloc_addr[dev];
  }
  float* xf = static_cast<float*>(base);
  float2* partial = reinterpret_cast<float2*>(static_cast<unsigned char*>(base) + xf_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  fs::Shape s{};
  s.H = hidden;
  s.V = vocab;
  s.eps = rms_eps;
  cudaError_t e = fs::launch_rmsnorm(x, rows, hidden,
                                     static_cast<const __nv_bfloat16*>(final_norm), rms_eps, xf, st);
  if (e == cudaSuccess)
    e = fs::launch_lm_head(xf, rows, s, static_cast<const __nv_bfloat16*>(embed), logits, argmax,
                           partial, n_part, nullptr, st);
  if (e != cudaSuccess) {
    set_error(std::string("fs_lm_head_argmax_noalloc: launch failed: ") + cudaGetErrorString(e));
    return FS_ERR_CUDA;
  }
  return FS_OK;
}
