// Handle structs behind the opaque fs_model / fs_kv of the C ABI, and the
// internal entry points the fast paths plug into.
#pragma once

#include <string>
#include <vector>

#include "fs_internal.h"

struct fs_model {
  fs_config cfg{};
  fs::Shape s{};
  bool q8 = false;
  int device = 0;
  int num_sms = 0;
  const __nv_bfloat16* embed = nullptr;       // caller-owned
  const __nv_bfloat16* final_norm = nullptr;  // caller-owned
  std::vector<fs::LayerDev> layers;           // caller-owned pointers
  // Library-owned buffers.
  float2* rope = nullptr;  // [max_pos][d/2] (cos, sin)
  int max_rows = 0;        // rows of one forward chunk
  float* h = nullptr;      // residual stream [max_rows, H]
  float* xn = nullptr;     // normalised rows [max_rows, max(H, nq*d, I)]
  float* qkv = nullptr;    // [max_rows, (nq+2nkv)*d]
  float* q = nullptr;      // rotated queries [max_rows, nq*d]
  float* o = nullptr;      // attention output [max_rows, nq*d]
  float* attn_part = nullptr;  // split-KV attention partials (attention_decode.cu)
  float* lm_scratch = nullptr; // logits of 5..16 rows when the caller passes none [16, V]
  float* gu = nullptr;     // gate||up [max_rows, 2I]
  float* act = nullptr;    // SwiGLU output [max_rows, I]
  float* xf = nullptr;     // final-normed rows [64, H]
  int32_t* tok = nullptr;  // staged token ids [max_rows]
  float2* partial = nullptr;  // LM-head argmax partials [64, n_part]
  int n_part = 0;
  int* err = nullptr;         // device error word
  int32_t* gen_tok = nullptr; // greedy ids
  int gen_cap = 0;
  void* scratch = nullptr;
  float* capture = nullptr;   // armed fs_debug_capture buffer
  int capture_max_rows = 0;
  int prefill_split = 1;
  unsigned long long* trace = nullptr;  // armed fs_debug_trace buffer
  void* extras = nullptr;     // persistent decode kernel state
  void* cl_extras = nullptr;  // cluster decode kernel state
  void* mega_extras = nullptr;  // row-split decode kernel state
  int decode_path = 0;        // fs_debug_decode_path: 0 auto, 1 cooperative kernel, 2 general
  void* tc_extras = nullptr;  // tensor-core prefill state
};

struct fs_kv {
  const fs_model* model = nullptr;
  int max_seqs = 0;
  int max_tokens = 0;
  int pages_per_seq = 0;
  int n_pages = 0;
  __nv_bfloat16* k = nullptr;
  __nv_bfloat16* v = nullptr;
  int32_t* block_table = nullptr;
  std::vector<int32_t> len;  // host-tracked lengths
};

namespace fs {

KVView kv_view(const fs_kv* kv);
int kv_capacity(const fs_kv* kv);
const char* set_error(const std::string& msg);
void model_free_buffers(fs_model* m);

fs_status init_extras(fs_model* m);
void release_extras(fs_model* m);
fs_status ensure_gen_buffer(fs_model* m, int n);

// The unfused general forward (any rows): see runtime.cu.
fs_status forward_general(fs_model* m, const fs_kv* kv, const RowMap& map, int rows,
                          const int32_t* tok, int head_first, float* logits, int32_t* argmax,
                          int capture_row0, int capture_rows, cudaStream_t st,
                          bool tensor_cores = false);

// One prefill chunk (consecutive positions of one sequence).
fs_status prefill_chunk(fs_model* m, const fs_kv* kv, const RowMap& map, int rows,
                        const int32_t* tok, int head_first, float* logits, int32_t* argmax,
                        int capture_row0, int capture_rows, cudaStream_t st);

// One decode step over a batch of sequences.
fs_status decode_rows(fs_model* m, const fs_kv* kv, const RowMap& map, int rows,
                      const int32_t* tok, float* logits, int32_t* argmax, cudaStream_t st);

// Persistent decode kernel (decode_fused.cu): set-up (transposed Wo / Wd,
// exchange buffers), release, reset after a device error, the debug wait
// limit, and one step of blocks [l0, l1) (+ the LM head) for 1..4 rows.
fs_status fused_init(fs_model* m);
void fused_release(fs_model* m);
void fused_reset(fs_model* m);
void fused_debug_wait(fs_model* m, unsigned long long wait_ns, int withhold_layer);
fs_status decode_fused(fs_model* m, const fs_kv* kv, const RowMap& map, int B, const int32_t* tok,
                       const float* h_in, float* h_out, int l0, int l1, bool run_head,
                       float* logits, int32_t* argmax, cudaStream_t stream);

// Row-split persistent decode kernel (decode_mega.cu): batch 1, the shapes
// whose ring holds a stage per consumer warp.
fs_status mega_init(fs_model* m);
void mega_release(fs_model* m);
void mega_reset(fs_model* m);
void mega_debug_wait(fs_model* m, unsigned long long wait_ns, int withhold_layer);
bool mega_eligible(const fs_model* m);
fs_status decode_mega(fs_model* m, const fs_kv* kv, const RowMap& map, int B, const int32_t* tok,
                      const float* h_in, float* h_out, int l0, int l1, bool run_head,
                      float* logits, int32_t* argmax, cudaStream_t stream);

// Cluster decode kernel (decode_cluster.cu): the same calls for the kernel
// that runs one 16-CTA cluster per kv head (bf16 weights, 1..4 rows).
fs_status cluster_init(fs_model* m);
void cluster_release(fs_model* m);
void cluster_reset(fs_model* m);
void cluster_debug_wait(fs_model* m, unsigned long long wait_ns, int withhold_layer);
bool cluster_eligible(const fs_model* m);
fs_status decode_cluster(fs_model* m, const fs_kv* kv, const RowMap& map, int B,
                         const int32_t* tok, const float* h_in, float* h_out, int l0, int l1,
                         bool run_head, float* logits, int32_t* argmax, cudaStream_t stream);
// The persistent kernel that fs_debug_decode_path selects: the cluster kernel,
// else the cooperative one; FS_ERR_UNSUPPORTED when neither covers the call.
fs_status decode_persistent(fs_model* m, const fs_kv* kv, const RowMap& map, int B,
                            const int32_t* tok, const float* h_in, float* h_out, int l0, int l1,
                            bool run_head, float* logits, int32_t* argmax, cudaStream_t stream);

// Tensor-core prefill (prefill_tc.cu): available for this model (prepares
// the fp16 weights on first use), one block on m->h, release.
bool tc_available(fs_model* m, cudaStream_t st);
fs_status layer_tc(fs_model* m, const fs_kv* kv, const RowMap& map, int rows, int l,
                   cudaStream_t st);
void tc_release(fs_model* m);
constexpr int kTcMinRows = 128;

// One block of the general path on m->h (rows described by map).
fs_status layer_general(fs_model* m, const fs_kv* kv, const RowMap& map, int rows, int l,
                        cudaStream_t st);

// The block kernels the prefill path uses for `rows` rows (debug entry point).
fs_status block_prefill_or_general(fs_model* m, const fs_kv* kv, const RowMap& map, int rows,
                                   int l, cudaStream_t st);

fs_status prefill_impl(fs_model* m, fs_kv* kv, int32_t seq, const int32_t* tokens, int32_t n,
                       float* logits, int32_t* argmax, cudaStream_t st);
fs_status decode_impl(fs_model* m, fs_kv* kv, const int32_t* seqs, const int32_t* tokens,
                      int32_t batch, float* logits, int32_t* argmax, cudaStream_t st);

}  // namespace fs
