// Internal declarations shared by the libfs CUDA sources (not part of the ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "fs.h"

namespace fs {

// Kernel launches issued by the library (fs_debug_kernel_launches).
void count_launches(int n = 1);

// Programmatic dependent launch. A kernel started with launch_pdl may begin
// while the kernel before it on the stream is still running: before reading
// anything an earlier kernel wrote (or writing what it reads) it calls
// pdl_wait(), which returns once the earlier grids have completed and their
// memory is visible; only immutable inputs (weights) may be read before it.
// pdl_trigger() lets the next kernel start early. Both are no-ops for a
// kernel launched without the attribute.
#ifdef __CUDACC__
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}
#endif

constexpr int kPage = 64;        // positions per KV page
constexpr int kMaxBatch = 64;    // rows of one decode step
constexpr int kMaxHeadDim = 128;

// Device error word values (fs_device_error).
constexpr int kErrToken = 1;
constexpr int kErrBounds = 2;
constexpr int kErrTimeout = 3;

// Index of each linear layer in LayerDev::w / LayerDev::s.
enum Lin { kWq = 0, kWk, kWv, kWo, kWg, kWu, kWd, kNumLin };

struct LayerDev {
  const void* w[kNumLin];   // bf16 [N,K] or int8 codes [N,K]
  const __half* s[kNumLin]; // Q8_0 scales [N,K/32] (nullptr for bf16)
  const __nv_bfloat16* attn_norm;
  const __nv_bfloat16* ffn_norm;
  const __nv_bfloat16* q_norm;
  const __nv_bfloat16* k_norm;
};

// Paged KV cache as the kernels see it. K and V pools are
// [layer][page][kv_head][slot 0..63][head_dim] bf16.
struct KVView {
  __nv_bfloat16* k;
  __nv_bfloat16* v;
  const int32_t* block_table;  // [max_seqs][pages_per_seq] physical page ids
  int32_t pages_per_seq;
  int32_t n_pages;
  int32_t n_kv_heads;
  int32_t head_dim;
  __host__ __device__ size_t layer_elems() const {
    return (size_t)n_pages * n_kv_heads * kPage * head_dim;
  }
  // Element offset of (layer, seq, pos, kv_head, 0).
  __device__ __forceinline__ size_t offset(int layer, int seq, int pos, int g) const {
    int page = block_table[(size_t)seq * pages_per_seq + pos / kPage];
    return (size_t)layer * layer_elems() +
           (((size_t)page * n_kv_heads + g) * kPage + (pos % kPage)) * head_dim;
  }
};

// Per-row (token) description of one forward call: which sequence it belongs
// to and at which position it sits.
struct RowInfo {
  int32_t seq;
  int32_t pos;
};

// Row map of one forward call, passed to kernels by value (no staging
// buffer): either `n_list` explicit (seq, pos) pairs (a decode batch) or, with
// n_list == 0, consecutive positions pos0, pos0+1, ... of one sequence seq0
// (a prefill chunk).
struct RowMap {
  int32_t n_list;
  int32_t seq0;
  int32_t pos0;
  int32_t seq[kMaxBatch];
  int32_t pos[kMaxBatch];
  __host__ __device__ __forceinline__ RowInfo get(int r) const {
    return n_list ? RowInfo{seq[r], pos[r]} : RowInfo{seq0, pos0 + r};
  }
};

struct Shape {
  int L, H, nq, nkv, d, I, V;
  float eps;
  int q_dim() const { return nq * d; }
  int kv_dim() const { return nkv * d; }
  int qkv_dim() const { return (nq + 2 * nkv) * d; }
};

// ---------------------------------------------------------------------------
// Kernel launchers (each defined next to its kernel). All return
// cudaGetLastError() after the launch.

cudaError_t launch_embed(const int32_t* tokens, int rows, const __nv_bfloat16* E, int H, int V,
                         float* h, int* err, cudaStream_t st);
cudaError_t launch_rmsnorm(const float* x, int rows, int H, const __nv_bfloat16* g, float eps,
                           float* out, cudaStream_t st, float* zero = nullptr, int zero_w = 0,
                           int zero_ld = 0);
// y = x . W^T over rows; epilogue: 0 store y, 1 y += into out (residual).
cudaError_t launch_gemv(const float* x, int rows, int K, const void* W, const __half* scales,
                        int N, float* out, int ldo, bool accumulate, cudaStream_t st);
// act[r, j] = silu(x . Wg[j]) * (x . Wu[j])
cudaError_t launch_gemv_swiglu(const float* x, int rows, int K, const void* Wg, const __half* sg,
                               const void* Wu, const __half* su, int N, float* act,
                               cudaStream_t st);
// Split-K weight streaming for 5..16 rows of bf16 weights (gemv_splitk.cu).
bool gemv_splitk_ok(int rows, int K, const __half* scales);
cudaError_t launch_gemv_splitk(const float* x, int rows, int K, const __nv_bfloat16* W, int N,
                               float* out, int ldo, bool accumulate, cudaStream_t st);
// The same for n (2 or 3) matrices of one input in one launch, written side by
// side from out0 (cleared first): q | k | v, gate | up.
cudaError_t launch_gemv_splitk_multi(const float* x, int rows, int K, int n,
                                     const __nv_bfloat16* const* W, const int* N, float* out0,
                                     int ldo, bool cleared, cudaStream_t st);
// y += silu(gate) * up times W^T, the SwiGLU computed while the input is
// staged: `gu` rows are [gate (K) | up (K)].
cudaError_t launch_gemv_splitk_swiglu(const float* gu, int rows, int K, const __nv_bfloat16* W,
                                      int N, float* out, int ldo, cudaStream_t st);
// Greedy id per row of fp32 logits [rows][V] (lowest id on exact ties).
cudaError_t launch_argmax_rows(const float* logits, int rows, int V, int32_t* argmax,
                               cudaStream_t st);
cudaError_t launch_gemm_simt(const float* A, int M, int K, const void* W, const __half* scales,
                             int N, float* C, int ldc, bool accumulate, cudaStream_t st);
cudaError_t launch_swiglu(const float* gu, int rows, int I, float* act, cudaStream_t st);
cudaError_t launch_qk_norm_rope_append(const float* qkv, int rows, const RowMap& map,
                                       const Shape& s, const __nv_bfloat16* q_norm,
                                       const __nv_bfloat16* k_norm, const float2* rope,
                                       float* q_out, KVView kv, int layer, cudaStream_t st);
cudaError_t launch_attention_simple(const float* q, int rows, const RowMap& map,
                                    const Shape& s, KVView kv, int layer, float* o,
                                    cudaStream_t st);
// Split-KV decode attention (rows <= 128, any positions); max_pos is the
// largest position among the rows, part the model's partial buffer.
bool attention_decode_supported(const Shape& s, int rows);
size_t attention_decode_part_floats(const Shape& s);
cudaError_t launch_attention_decode(const float* q, int rows, const RowMap& map, int max_pos,
                                    const Shape& s, KVView kv, int layer, float* part, float* o,
                                    int num_sms, cudaStream_t st);
// x: final-normed rows fp32 [rows, H]; partial: scratch of rows * n_part float2.
cudaError_t launch_lm_head(const float* xf, int rows, const Shape& s, const __nv_bfloat16* E,
                           float* logits, int32_t* argmax, float2* partial, int n_part, int* err,
                           cudaStream_t st);
// Seeded sampling of one id per row (sample.cu): temperature > 0, top_k (0 =
// off), top_p in (0, 1]; the draw of row r uses Philox4x32-10 at counter
// (step, r).
cudaError_t launch_sample(const float* logits, int rows, int V, float temperature, int top_k,
                          float top_p, unsigned long long seed, unsigned long long step,
                          int32_t* out, cudaStream_t st);
cudaError_t launch_dequant_q8_0(const int8_t* codes, const __half* scales, int n, int k,
                                float* out, cudaStream_t st);
cudaError_t launch_kv_copy(KVView kv, int seq, int layer, int pos0, int n, __nv_bfloat16* k,
                           __nv_bfloat16* v, bool import, cudaStream_t st);

}  // namespace fs
