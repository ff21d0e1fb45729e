// Chooses the kernel sequence for each forward call.
#include <atomic>

#include "runtime.h"

namespace fs {

fs_status init_extras(fs_model* m) {
  fs_status s = fused_init(m);
  if (s != FS_OK) return s;
  if ((s = mega_init(m)) != FS_OK) return s;
  return cluster_init(m);
}

void release_extras(fs_model* m) {
  cluster_release(m);
  mega_release(m);
  fused_release(m);
  tc_release(m);
}

fs_status decode_persistent(fs_model* m, const fs_kv* kv, const RowMap& map, int B,
                            const int32_t* tok, const float* h_in, float* h_out, int l0, int l1,
                            bool run_head, float* logits, int32_t* argmax, cudaStream_t stream) {
  const int path = m->decode_path;
  if (path == 2) return FS_ERR_UNSUPPORTED;
  if (path == 3 || (path == 0 && B == 1)) {
    fs_status s = decode_mega(m, kv, map, B, tok, h_in, h_out, l0, l1, run_head, logits, argmax,
                              stream);
    if (s != FS_ERR_UNSUPPORTED || path == 3) return s;
  }
  if (path == 0 || path == 4) {
    fs_status s = decode_cluster(m, kv, map, B, tok, h_in, h_out, l0, l1, run_head, logits,
                                 argmax, stream);
    if (s != FS_ERR_UNSUPPORTED || path == 4) return s;
  }
  return decode_fused(m, kv, map, B, tok, h_in, h_out, l0, l1, run_head, logits, argmax, stream);
}

fs_status ensure_gen_buffer(fs_model* m, int n) {
  if (n <= m->gen_cap) return FS_OK;
  if (m->gen_tok) cudaFree(m->gen_tok);
  m->gen_tok = nullptr;
  m->gen_cap = 0;
  if (cudaMalloc(&m->gen_tok, (size_t)n * sizeof(int32_t)) != cudaSuccess) {
    cudaGetLastError();
    set_error("out of device memory for greedy ids");
    return FS_ERR_OOM;
  }
  m->gen_cap = n;
  return FS_OK;
}

// Chunks of at least 128 rows run their GEMMs on the tensor cores.
fs_status prefill_chunk(fs_model* m, const fs_kv* kv, const RowMap& map, int rows,
                        const int32_t* tok, int head_first, float* logits, int32_t* argmax,
                        int capture_row0, int capture_rows, cudaStream_t st) {
  const bool tc = rows >= kTcMinRows && tc_available(m, st);
  return forward_general(m, kv, map, rows, tok, head_first, logits, argmax, capture_row0,
                         capture_rows, st, tc);
}

fs_status block_prefill_or_general(fs_model* m, const fs_kv* kv, const RowMap& map, int rows,
                                   int l, cudaStream_t st) {
  if (rows >= kTcMinRows && tc_available(m, st)) return layer_tc(m, kv, map, rows, l, st);
  return layer_general(m, kv, map, rows, l, st);
}

fs_status decode_rows(fs_model* m, const fs_kv* kv, const RowMap& map, int rows,
                      const int32_t* tok, float* logits, int32_t* argmax, cudaStream_t st) {
  // Distinct sequences (checked by the caller), at most 4: the persistent kernel.
  fs_status s = decode_persistent(m, kv, map, rows, tok, nullptr, nullptr, 0, m->s.L, true,
                                  logits, argmax, st);
  if (s != FS_ERR_UNSUPPORTED) return s;
  return forward_general(m, kv, map, rows, tok, 0, logits, argmax, 0, rows, st);
}

}  // namespace fs

namespace fs {
namespace {
std::atomic<uint64_t> g_launches{0};
}
void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }
}  // namespace fs

extern "C" uint64_t fs_debug_kernel_launches(void) { return fs::g_launches.load(); }
