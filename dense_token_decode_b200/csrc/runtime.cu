// libfs runtime: model and KV-cache handles, argument validation, the forward
// orchestration behind fs_prefill / fs_decode_step, and the greedy loop.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "fs_internal.h"
#include "runtime.h"

namespace {

thread_local std::string g_last_error;

fs_status fail(fs_status code, const std::string& msg) {
  g_last_error = msg;
  return code;
}

fs_status cuda_fail(cudaError_t e, const char* what) {
  return fail(FS_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

#define FS_CUDA(call)                                   \
  do {                                                  \
    cudaError_t e_ = (call);                            \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 1 = device (or managed) memory, 0 = host memory, -1 = unknown pointer.
int pointer_kind(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) ? 1 : 0;
}

fs_status check_device_ptr(const void* p, const char* name) {
  if (!p) return fail(FS_ERR_NULL, std::string(name) + " is NULL");
  if (!aligned16(p)) return fail(FS_ERR_ALIGN, std::string(name) + " is not 16-byte aligned");
  if (pointer_kind(p) != 1) return fail(FS_ERR_INVALID, std::string(name) + " is not device memory");
  return FS_OK;
}

template <typename T>
fs_status dev_alloc(T** p, size_t count, const char* what) {
  *p = nullptr;
  if (count == 0) count = 1;
  if (cudaMalloc(reinterpret_cast<void**>(p), count * sizeof(T)) != cudaSuccess) {
    cudaGetLastError();
    *p = nullptr;
    return fail(FS_ERR_OOM, std::string("out of device memory for ") + what);
  }
  return FS_OK;
}

}  // namespace

// ---------------------------------------------------------------------------

namespace fs {

void model_free_buffers(fs_model* m) {
  void* bufs[] = {m->rope, m->h,   m->xn,  m->qkv,     m->q,   m->o,       m->gu,
                  m->act,  m->xf,  m->tok, m->partial, m->err, m->gen_tok, m->scratch,
                  m->attn_part, m->lm_scratch};
  for (void* b : bufs)
    if (b) cudaFree(b);
  release_extras(m);
}

const char* set_error(const std::string& msg) {
  g_last_error = msg;
  return g_last_error.c_str();
}

}  // namespace fs

using fs::KVView;
using fs::RowMap;

// ---------------------------------------------------------------------------
// Model

extern "C" fs_status fs_model_create(const fs_config* cfg, const fs_weights* w, fs_model** out) {
  if (!out) return fail(FS_ERR_NULL, "out is NULL");
  *out = nullptr;
  if (!cfg || !w) return fail(FS_ERR_NULL, "config or weights is NULL");
  const fs_config c = *cfg;
  if (c.n_layers <= 0 || c.hidden <= 0 || c.n_q_heads <= 0 || c.n_kv_heads <= 0 ||
      c.head_dim <= 0 || c.ffn <= 0 || c.vocab <= 0 || c.max_pos <= 0 || c.max_pos > (1 << 20))
    return fail(FS_ERR_INVALID, "config sizes must be positive (max_pos <= 2^20)");
  if (c.n_q_heads % c.n_kv_heads) return fail(FS_ERR_INVALID, "n_q_heads % n_kv_heads != 0");
  if (!(c.rms_eps > 0.f) || !(c.rope_theta > 1.0))
    return fail(FS_ERR_INVALID, "rms_eps must be > 0 and rope_theta > 1");
  if (c.weight_format != FS_WEIGHT_BF16 && c.weight_format != FS_WEIGHT_Q8_0)
    return fail(FS_ERR_INVALID, "unknown weight_format");
  if (c.head_dim != 64 && c.head_dim != 128)
    return fail(FS_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (c.hidden % 64 || c.ffn % 64 || (c.n_q_heads * c.head_dim) % 64)
    return fail(FS_ERR_UNSUPPORTED, "hidden, ffn and n_q_heads*head_dim must be multiples of 64");
  if (c.n_q_heads + c.n_kv_heads > 32)
    return fail(FS_ERR_UNSUPPORTED, "n_q_heads + n_kv_heads must be <= 32");

  fs_status st;
  if ((st = check_device_ptr(w->embed, "embed")) != FS_OK) return st;
  if ((st = check_device_ptr(w->final_norm, "final_norm")) != FS_OK) return st;
  if (!w->layers) return fail(FS_ERR_NULL, "layers is NULL");
  const bool q8 = c.weight_format == FS_WEIGHT_Q8_0;
  std::vector<fs::LayerDev> layers(c.n_layers);
  for (int l = 0; l < c.n_layers; ++l) {
    const fs_layer_weights& lw = w->layers[l];
    const fs_linear* lin[fs::kNumLin] = {&lw.wq, &lw.wk, &lw.wv, &lw.wo, &lw.wg, &lw.wu, &lw.wd};
    static const char* names[fs::kNumLin] = {"wq", "wk", "wv", "wo", "wg", "wu", "wd"};
    for (int i = 0; i < fs::kNumLin; ++i) {
      const std::string nm = "layer " + std::to_string(l) + " " + names[i];
      if ((st = check_device_ptr(lin[i]->data, nm.c_str())) != FS_OK) return st;
      if (q8) {
        if ((st = check_device_ptr(lin[i]->scales, (nm + " scales").c_str())) != FS_OK) return st;
      } else if (lin[i]->scales) {
        return fail(FS_ERR_INVALID, nm + ": bf16 weights take no scales");
      }
      layers[l].w[i] = lin[i]->data;
      layers[l].s[i] = static_cast<const __half*>(q8 ? lin[i]->scales : nullptr);
    }
    const void* norms[4] = {lw.attn_norm, lw.ffn_norm, lw.q_norm, lw.k_norm};
    for (int i = 0; i < 4; ++i)
      if ((st = check_device_ptr(norms[i], "norm gain")) != FS_OK) return st;
    layers[l].attn_norm = static_cast<const __nv_bfloat16*>(lw.attn_norm);
    layers[l].ffn_norm = static_cast<const __nv_bfloat16*>(lw.ffn_norm);
    layers[l].q_norm = static_cast<const __nv_bfloat16*>(lw.q_norm);
    layers[l].k_norm = static_cast<const __nv_bfloat16*>(lw.k_norm);
  }

  fs_model* m = new fs_model();
  m->cfg = c;
  m->s = fs::Shape{c.n_layers, c.hidden, c.n_q_heads, c.n_kv_heads, c.head_dim,
                   c.ffn,      c.vocab,  c.rms_eps};
  m->q8 = q8;
  m->embed = static_cast<const __nv_bfloat16*>(w->embed);
  m->final_norm = static_cast<const __nv_bfloat16*>(w->final_norm);
  m->layers = layers;
  cudaGetDevice(&m->device);
  cudaDeviceGetAttribute(&m->num_sms, cudaDevAttrMultiProcessorCount, m->device);
  m->max_rows = std::max(std::min(c.max_pos, 2048), fs::kMaxBatch);
  m->n_part = 4 * m->num_sms;
  const fs::Shape& s = m->s;
  const size_t R = m->max_rows;

  // RoPE cos/sin table [max_pos][d/2], angle = pos * theta^(-2i/d) in fp64.
  {
    const int half = c.head_dim / 2;
    std::vector<float2> tab((size_t)c.max_pos * half);
    for (int i = 0; i < half; ++i) {
      const double inv_freq = std::pow(c.rope_theta, -2.0 * i / c.head_dim);
      for (int p = 0; p < c.max_pos; ++p) {
        const double a = (double)p * inv_freq;
        tab[(size_t)p * half + i] = make_float2((float)std::cos(a), (float)std::sin(a));
      }
    }
    if ((st = dev_alloc(&m->rope, tab.size(), "rope table")) != FS_OK) {
      fs::model_free_buffers(m);
      delete m;
      return st;
    }
    cudaMemcpy(m->rope, tab.data(), tab.size() * sizeof(float2), cudaMemcpyHostToDevice);
  }
  const size_t widest = std::max({(size_t)s.H, (size_t)s.q_dim(), (size_t)s.I});
  if ((st = dev_alloc(&m->h, R * s.H, "workspace")) != FS_OK ||
      (st = dev_alloc(&m->xn, R * widest, "workspace")) != FS_OK ||
      (st = dev_alloc(&m->qkv, R * s.qkv_dim(), "workspace")) != FS_OK ||
      (st = dev_alloc(&m->q, R * s.q_dim(), "workspace")) != FS_OK ||
      (st = dev_alloc(&m->o, R * s.q_dim(), "workspace")) != FS_OK ||
      (st = dev_alloc(&m->attn_part, fs::attention_decode_part_floats(s), "workspace")) != FS_OK ||
      (st = dev_alloc(&m->lm_scratch, (size_t)16 * s.V, "workspace")) != FS_OK ||
      (st = dev_alloc(&m->gu, R * 2 * s.I, "workspace")) != FS_OK ||
      (st = dev_alloc(&m->act, R * s.I, "workspace")) != FS_OK ||
      (st = dev_alloc(&m->xf, (size_t)fs::kMaxBatch * s.H, "workspace")) != FS_OK ||
      (st = dev_alloc(&m->tok, R, "workspace")) != FS_OK ||
      (st = dev_alloc(&m->partial, (size_t)fs::kMaxBatch * m->n_part, "workspace")) != FS_OK ||
      (st = dev_alloc(&m->err, 1, "error word")) != FS_OK) {
    fs::model_free_buffers(m);
    delete m;
    return st;
  }
  cudaMemset(m->err, 0, sizeof(int));
  if ((st = fs::init_extras(m)) != FS_OK) {
    fs::model_free_buffers(m);
    delete m;
    return st;
  }
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    fs::model_free_buffers(m);
    delete m;
    return cuda_fail(e, "model set-up");
  }
  *out = m;
  g_last_error.clear();
  return FS_OK;
}

extern "C" void fs_model_destroy(fs_model* m) {
  if (!m) return;
  fs::model_free_buffers(m);
  delete m;
}

extern "C" fs_status fs_set_prefill_split(fs_model* m, int32_t split) {
  if (!m) return fail(FS_ERR_NULL, "model is NULL");
  if (split != 0 && split != 1) return fail(FS_ERR_INVALID, "split must be 0 or 1");
  m->prefill_split = split;
  return FS_OK;
}

extern "C" fs_status fs_device_error(fs_model* m, int32_t* code) {
  if (!m || !code) return fail(FS_ERR_NULL, "model or code is NULL");
  int v = 0;
  FS_CUDA(cudaMemcpy(&v, m->err, sizeof(int), cudaMemcpyDeviceToHost));
  FS_CUDA(cudaMemset(m->err, 0, sizeof(int)));
  if (v) {
    fs::fused_reset(m);
    fs::cluster_reset(m);
    fs::mega_reset(m);
  }
  *code = v;
  return FS_OK;
}

// ---------------------------------------------------------------------------
// KV cache

extern "C" fs_status fs_kv_alloc(const fs_model* m, int32_t max_seqs, int32_t max_tokens,
                                 fs_kv** out) {
  if (!out) return fail(FS_ERR_NULL, "out is NULL");
  *out = nullptr;
  if (!m) return fail(FS_ERR_NULL, "model is NULL");
  if (max_seqs <= 0 || max_tokens <= 0 || max_seqs > (1 << 16))
    return fail(FS_ERR_INVALID, "max_seqs and max_tokens_per_seq must be positive");
  const int pps = (max_tokens + fs::kPage - 1) / fs::kPage;
  const long long n_pages = (long long)pps * max_seqs;
  if (n_pages > (1LL << 30)) return fail(FS_ERR_INVALID, "KV cache too large");
  fs_kv* kv = new fs_kv();
  kv->model = m;
  kv->max_seqs = max_seqs;
  kv->max_tokens = max_tokens;
  kv->pages_per_seq = pps;
  kv->n_pages = (int)n_pages;
  kv->len.assign(max_seqs, 0);
  const size_t elems =
      (size_t)m->s.L * n_pages * m->s.nkv * fs::kPage * m->s.d;
  fs_status st;
  if ((st = dev_alloc(&kv->k, elems, "KV pages")) != FS_OK ||
      (st = dev_alloc(&kv->v, elems, "KV pages")) != FS_OK ||
      (st = dev_alloc(&kv->block_table, (size_t)n_pages, "block table")) != FS_OK) {
    fs_kv_free(kv);
    return st;
  }
  // Attention kernels read whole pages and weight the slots past a sequence's
  // length by exact zeros: those slots must hold finite values.
  if (cudaMemset(kv->k, 0, elems * sizeof(__nv_bfloat16)) != cudaSuccess ||
      cudaMemset(kv->v, 0, elems * sizeof(__nv_bfloat16)) != cudaSuccess) {
    fs_kv_free(kv);
    return cuda_fail(cudaGetLastError(), "KV page clear");
  }
  // Page i of sequence s is physical page n_pages-1-(s*pps+i): the kernels
  // always go through the table, never assume contiguity.
  std::vector<int32_t> table(n_pages);
  for (long long i = 0; i < n_pages; ++i) table[i] = (int32_t)(n_pages - 1 - i);
  cudaError_t e = cudaMemcpy(kv->block_table, table.data(), n_pages * sizeof(int32_t),
                             cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    fs_kv_free(kv);
    return cuda_fail(e, "block table upload");
  }
  *out = kv;
  return FS_OK;
}

extern "C" void fs_kv_free(fs_kv* kv) {
  if (!kv) return;
  if (kv->k) cudaFree(kv->k);
  if (kv->v) cudaFree(kv->v);
  if (kv->block_table) cudaFree(kv->block_table);
  delete kv;
}

namespace fs {
KVView kv_view(const fs_kv* kv) {
  KVView v;
  v.k = kv->k;
  v.v = kv->v;
  v.block_table = kv->block_table;
  v.pages_per_seq = kv->pages_per_seq;
  v.n_pages = kv->n_pages;
  v.n_kv_heads = kv->model->s.nkv;
  v.head_dim = kv->model->s.d;
  return v;
}

int kv_capacity(const fs_kv* kv) { return std::min(kv->max_tokens, kv->model->cfg.max_pos); }
}  // namespace fs

extern "C" fs_status fs_kv_reset(fs_kv* kv, int32_t seq) {
  if (!kv) return fail(FS_ERR_NULL, "kv is NULL");
  if (seq < 0 || seq >= kv->max_seqs) return fail(FS_ERR_SEQ, "sequence out of range");
  FS_CUDA(cudaDeviceSynchronize());
  kv->len[seq] = 0;
  return FS_OK;
}

extern "C" fs_status fs_kv_length(const fs_kv* kv, int32_t seq, int32_t* len) {
  if (!kv || !len) return fail(FS_ERR_NULL, "kv or len is NULL");
  if (seq < 0 || seq >= kv->max_seqs) return fail(FS_ERR_SEQ, "sequence out of range");
  *len = kv->len[seq];
  return FS_OK;
}

extern "C" fs_status fs_kv_set_length(fs_kv* kv, int32_t seq, int32_t len) {
  if (!kv) return fail(FS_ERR_NULL, "kv is NULL");
  if (seq < 0 || seq >= kv->max_seqs) return fail(FS_ERR_SEQ, "sequence out of range");
  if (len < 0 || len > fs::kv_capacity(kv)) return fail(FS_ERR_CONTEXT, "length beyond capacity");
  kv->len[seq] = len;
  return FS_OK;
}

static fs_status kv_copy_checked(const fs_kv* kv, int32_t seq, int32_t layer, int32_t pos0,
                                 int32_t n, const void* k, const void* v, void* stream,
                                 bool import) {
  if (!kv) return fail(FS_ERR_NULL, "kv is NULL");
  if (seq < 0 || seq >= kv->max_seqs) return fail(FS_ERR_SEQ, "sequence out of range");
  if (layer < 0 || layer >= kv->model->s.L) return fail(FS_ERR_INVALID, "layer out of range");
  if (n < 0 || pos0 < 0) return fail(FS_ERR_INVALID, "negative position or count");
  if ((long long)pos0 + n > fs::kv_capacity(kv)) return fail(FS_ERR_CONTEXT, "beyond KV capacity");
  if (n == 0) return FS_OK;
  fs_status st;
  if ((st = check_device_ptr(k, "k")) != FS_OK || (st = check_device_ptr(v, "v")) != FS_OK)
    return st;
  FS_CUDA(fs::launch_kv_copy(fs::kv_view(kv), seq, layer, pos0, n,
                             const_cast<__nv_bfloat16*>(static_cast<const __nv_bfloat16*>(k)),
                             const_cast<__nv_bfloat16*>(static_cast<const __nv_bfloat16*>(v)),
                             import, static_cast<cudaStream_t>(stream)));
  return FS_OK;
}

extern "C" fs_status fs_kv_import(fs_kv* kv, int32_t seq, int32_t layer, int32_t pos0, int32_t n,
                                  const void* k, const void* v, void* stream) {
  return kv_copy_checked(kv, seq, layer, pos0, n, k, v, stream, true);
}

extern "C" fs_status fs_kv_export(const fs_kv* kv, int32_t seq, int32_t layer, int32_t pos0,
                                  int32_t n, void* k, void* v, void* stream) {
  return kv_copy_checked(kv, seq, layer, pos0, n, k, v, stream, false);
}

// ---------------------------------------------------------------------------
// Forward

namespace fs {

// y (+)= x . W^T for `rows` rows, the GEMV for a few rows, the tiled GEMM beyond.
static cudaError_t linear(const fs_model* m, const float* x, int rows, int K, int layer, Lin which,
                          int N, float* out, int ldo, bool acc, cudaStream_t st) {
  const LayerDev& L = m->layers[layer];
  if (rows > 4 && gemv_splitk_ok(rows, K, L.s[which]))
    return launch_gemv_splitk(x, rows, K, static_cast<const __nv_bfloat16*>(L.w[which]), N, out,
                              ldo, acc, st);
  if (rows <= 16) return launch_gemv(x, rows, K, L.w[which], L.s[which], N, out, ldo, acc, st);
  return launch_gemm_simt(x, rows, K, L.w[which], L.s[which], N, out, ldo, acc, st);
}

// One block over m->h (in place): RMSNorm, Q/K/V, head norm + RoPE + KV
// append, attention, O + residual, RMSNorm, SwiGLU MLP + residual.
fs_status layer_general(fs_model* m, const fs_kv* kv, const RowMap& map, int rows, int l,
                      cudaStream_t st) {
  const Shape& s = m->s;
  const KVView kvv = kv_view(kv);
  const int H = s.H, qd = s.q_dim(), kvd = s.kv_dim(), qkvd = s.qkv_dim();
  const LayerDev& Lw = m->layers[l];
  const bool splitk = rows > 4 && gemv_splitk_ok(rows, H, Lw.s[kWq]);
  // the split-K products accumulate: their output blocks are cleared by the
  // RMSNorm kernel before them
  FS_CUDA(launch_rmsnorm(m->h, rows, H, Lw.attn_norm, s.eps, m->xn, st, splitk ? m->qkv : nullptr,
                         qkvd, qkvd));
  if (splitk) {
    // q | k | v in one launch
    const __nv_bfloat16* W3[3] = {static_cast<const __nv_bfloat16*>(Lw.w[kWq]),
                                  static_cast<const __nv_bfloat16*>(Lw.w[kWk]),
                                  static_cast<const __nv_bfloat16*>(Lw.w[kWv])};
    const int N3[3] = {qd, kvd, kvd};
    FS_CUDA(launch_gemv_splitk_multi(m->xn, rows, H, 3, W3, N3, m->qkv, qkvd, true, st));
  } else {
    FS_CUDA(linear(m, m->xn, rows, H, l, kWq, qd, m->qkv, qkvd, false, st));
    FS_CUDA(linear(m, m->xn, rows, H, l, kWk, kvd, m->qkv + qd, qkvd, false, st));
    FS_CUDA(linear(m, m->xn, rows, H, l, kWv, kvd, m->qkv + qd + kvd, qkvd, false, st));
  }
  FS_CUDA(launch_qk_norm_rope_append(m->qkv, rows, map, s, Lw.q_norm, Lw.k_norm, m->rope, m->q,
                                     kvv, l, st));
  if (attention_decode_supported(s, rows)) {
    int max_pos = 0;
    for (int r = 0; r < rows; ++r) max_pos = std::max(max_pos, map.get(r).pos);
    FS_CUDA(launch_attention_decode(m->q, rows, map, max_pos, s, kvv, l, m->attn_part, m->o,
                                    m->num_sms, st));
  } else {
    FS_CUDA(launch_attention_simple(m->q, rows, map, s, kvv, l, m->o, st));
  }
  FS_CUDA(linear(m, m->o, rows, qd, l, kWo, H, m->h, H, true, st));
  const bool splitk_mlp = rows > 4 && gemv_splitk_ok(rows, H, Lw.s[kWg]) &&
                         gemv_splitk_ok(rows, s.I, Lw.s[kWd]);
  FS_CUDA(launch_rmsnorm(m->h, rows, H, Lw.ffn_norm, s.eps, m->xn, st,
                         splitk_mlp ? m->gu : nullptr, 2 * s.I, 2 * s.I));
  if (splitk_mlp) {
    // gate | up in one launch, then down with the SwiGLU computed as its input
    // is staged
    const __nv_bfloat16* W2[2] = {static_cast<const __nv_bfloat16*>(Lw.w[kWg]),
                                  static_cast<const __nv_bfloat16*>(Lw.w[kWu])};
    const int N2[2] = {s.I, s.I};
    FS_CUDA(launch_gemv_splitk_multi(m->xn, rows, H, 2, W2, N2, m->gu, 2 * s.I, true, st));
    FS_CUDA(launch_gemv_splitk_swiglu(m->gu, rows, s.I,
                                      static_cast<const __nv_bfloat16*>(Lw.w[kWd]), H, m->h, H,
                                      st));
    return FS_OK;
  }
  if (rows <= 16 && !(rows > 4 && gemv_splitk_ok(rows, H, Lw.s[kWg]))) {
    FS_CUDA(launch_gemv_swiglu(m->xn, rows, H, Lw.w[kWg], Lw.s[kWg], Lw.w[kWu], Lw.s[kWu], s.I,
                               m->act, st));
  } else {
    FS_CUDA(linear(m, m->xn, rows, H, l, kWg, s.I, m->gu, 2 * s.I, false, st));
    FS_CUDA(linear(m, m->xn, rows, H, l, kWu, s.I, m->gu + s.I, 2 * s.I, false, st));
    FS_CUDA(launch_swiglu(m->gu, rows, s.I, m->act, st));
  }
  FS_CUDA(linear(m, m->act, rows, s.I, l, kWd, H, m->h, H, true, st));
  return FS_OK;
}

// The general forward over `rows` rows described by `map`, tokens on the
// device. Writes logits/argmax for the rows selected by `head_rows`:
// head_first .. rows-1 (prefill: the last row; decode: every row).
fs_status forward_general(fs_model* m, const fs_kv* kv, const RowMap& map, int rows,
                          const int32_t* tok, int head_first, float* logits, int32_t* argmax,
                          int capture_row0, int capture_rows, cudaStream_t st, bool tensor_cores) {
  (void)capture_rows;
  const Shape& s = m->s;
  const int H = s.H;
  FS_CUDA(launch_embed(tok, rows, m->embed, H, s.V, m->h, m->err, st));
  auto capture = [&](int slot) -> cudaError_t {
    if (!m->capture) return cudaSuccess;
    const int n = std::min(rows, m->capture_max_rows - capture_row0);
    if (n <= 0) return cudaSuccess;
    return cudaMemcpyAsync(m->capture + ((size_t)slot * m->capture_max_rows + capture_row0) * H, m->h,
                           (size_t)n * H * sizeof(float), cudaMemcpyDeviceToDevice, st);
  };
  FS_CUDA(capture(0));
  for (int l = 0; l < s.L; ++l) {
    fs_status ls = tensor_cores ? layer_tc(m, kv, map, rows, l, st)
                                : layer_general(m, kv, map, rows, l, st);
    if (ls != FS_OK) return ls;
    FS_CUDA(capture(l + 1));
  }
  const int nh = rows - head_first;
  if (nh > 0 && (logits || argmax)) {
    FS_CUDA(launch_rmsnorm(m->h + (size_t)head_first * H, nh, H, m->final_norm, s.eps, m->xf, st));
    if (nh > 4 && gemv_splitk_ok(nh, H, nullptr)) {
      // 5..16 rows: split-K streaming of the tied embedding into the logits
      // (the caller's, or the model's scratch), then the greedy pass.
      float* lg = logits ? logits : m->lm_scratch;
      FS_CUDA(launch_gemv_splitk(m->xf, nh, H, m->embed, s.V, lg, s.V, false, st));
      if (argmax) FS_CUDA(launch_argmax_rows(lg, nh, s.V, argmax, st));
    } else {
      FS_CUDA(launch_lm_head(m->xf, nh, s, m->embed, logits, argmax, m->partial, m->n_part,
                             m->err, st));
    }
  }
  return FS_OK;
}

}  // namespace fs

// Copy (host) or adopt (device) a token array for a forward call.
static fs_status stage_tokens(fs_model* m, const int32_t* tokens, int n, int32_t* dst,
                              const int32_t** dev_tokens, cudaStream_t st) {
  if (!tokens) return fail(FS_ERR_NULL, "tokens is NULL");
  if (pointer_kind(tokens) == 1) {
    if (!aligned16(tokens) && ((reinterpret_cast<uintptr_t>(tokens) & 3u) != 0))
      return fail(FS_ERR_ALIGN, "device tokens are not 4-byte aligned");
    *dev_tokens = tokens;
    return FS_OK;
  }
  for (int i = 0; i < n; ++i)
    if (tokens[i] < 0 || tokens[i] >= m->s.V)
      return fail(FS_ERR_TOKEN, "token id " + std::to_string(tokens[i]) + " at index " +
                                    std::to_string(i) + " is outside [0, vocab)");
  FS_CUDA(cudaMemcpyAsync(dst, tokens, (size_t)n * sizeof(int32_t), cudaMemcpyHostToDevice, st));
  *dev_tokens = dst;
  return FS_OK;
}

static fs_status check_out_ptr(const void* p, const char* name) {
  if (!p) return FS_OK;
  return check_device_ptr(p, name);
}

// int32 outputs only need their natural 4-byte alignment.
static fs_status check_i32_out(const void* p, const char* name) {
  if (!p) return FS_OK;
  if (reinterpret_cast<uintptr_t>(p) & 3u)
    return fail(FS_ERR_ALIGN, std::string(name) + " is not 4-byte aligned");
  if (pointer_kind(p) != 1) return fail(FS_ERR_INVALID, std::string(name) + " is not device memory");
  return FS_OK;
}

namespace fs {

fs_status prefill_impl(fs_model* m, fs_kv* kv, int32_t seq, const int32_t* tokens, int32_t n,
                       float* logits, int32_t* argmax, cudaStream_t st) {
  if (!m || !kv) return fail(FS_ERR_NULL, "model or kv is NULL");
  if (kv->model != m) return fail(FS_ERR_INVALID, "kv belongs to another model");
  if (n <= 0) return fail(FS_ERR_EMPTY, "prefill needs at least one token");
  if (seq < 0 || seq >= kv->max_seqs) return fail(FS_ERR_SEQ, "sequence out of range");
  fs_status s;
  if ((s = check_out_ptr(logits, "logits_out")) != FS_OK) return s;
  if ((s = check_i32_out(argmax, "argmax_out")) != FS_OK) return s;
  const int pos0 = kv->len[seq];
  if ((long long)pos0 + n > kv_capacity(kv))
    return fail(FS_ERR_CONTEXT, "prefill would exceed max_pos or the KV capacity");
  const int32_t* dev_tok = nullptr;
  const bool on_device = pointer_kind(tokens) == 1;
  for (int c0 = 0; c0 < n; c0 += m->max_rows) {
    const int rows = std::min(m->max_rows, n - c0);
    if ((s = stage_tokens(m, tokens + c0, rows, m->tok, &dev_tok, st)) != FS_OK) return s;
    (void)on_device;
    RowMap map{};
    map.n_list = 0;
    map.seq0 = seq;
    map.pos0 = pos0 + c0;
    const bool last = c0 + rows == n;
    if ((s = prefill_chunk(m, kv, map, rows, dev_tok, last ? rows - 1 : rows,
                           last ? logits : nullptr, last ? argmax : nullptr, c0, n, st)) != FS_OK)
      return s;
  }
  kv->len[seq] = pos0 + n;
  if (m->capture) m->capture = nullptr;
  return FS_OK;
}

fs_status decode_impl(fs_model* m, fs_kv* kv, const int32_t* seqs, const int32_t* tokens,
                      int32_t batch, float* logits, int32_t* argmax, cudaStream_t st) {
  if (!m || !kv) return fail(FS_ERR_NULL, "model or kv is NULL");
  if (kv->model != m) return fail(FS_ERR_INVALID, "kv belongs to another model");
  if (batch <= 0) return fail(FS_ERR_EMPTY, "decode needs at least one sequence");
  if (batch > kMaxBatch) return fail(FS_ERR_INVALID, "batch must be <= 64");
  if (!seqs) return fail(FS_ERR_NULL, "seqs is NULL");
  fs_status s;
  if ((s = check_out_ptr(logits, "logits_out")) != FS_OK) return s;
  if ((s = check_i32_out(argmax, "argmax_out")) != FS_OK) return s;
  RowMap map{};
  map.n_list = batch;
  const int cap = kv_capacity(kv);
  for (int b = 0; b < batch; ++b) {
    const int q = seqs[b];
    if (q < 0 || q >= kv->max_seqs) return fail(FS_ERR_SEQ, "sequence out of range");
    for (int c = 0; c < b; ++c)
      if (seqs[c] == q) return fail(FS_ERR_SEQ, "a sequence appears twice in one batch");
    if (kv->len[q] + 1 > cap)
      return fail(FS_ERR_CONTEXT, "decode would exceed max_pos or the KV capacity");
    map.seq[b] = q;
    map.pos[b] = kv->len[q];
  }
  const int32_t* dev_tok = nullptr;
  if ((s = stage_tokens(m, tokens, batch, m->tok, &dev_tok, st)) != FS_OK) return s;
  if ((s = decode_rows(m, kv, map, batch, dev_tok, logits, argmax, st)) != FS_OK) return s;
  for (int b = 0; b < batch; ++b) kv->len[seqs[b]] += 1;
  if (m->capture) m->capture = nullptr;
  return FS_OK;
}

// A mixed batch: segment i appends n_tokens[i] ids of sequence seqs[i]. The
// rows go through one general forward, ordered so that every segment's last
// row comes at the end (in segment order): the LM head then runs on exactly
// those rows. Every row's K/V is appended before any row attends, so the
// order does not change what a row sees.
fs_status batch_impl(fs_model* m, fs_kv* kv, const int32_t* seqs, const int32_t* n_tokens,
                     int32_t n_seqs, const int32_t* tokens, float* logits, int32_t* argmax,
                     cudaStream_t st) {
  if (!m || !kv) return fail(FS_ERR_NULL, "model or kv is NULL");
  if (kv->model != m) return fail(FS_ERR_INVALID, "kv belongs to another model");
  if (!seqs || !n_tokens || !tokens) return fail(FS_ERR_NULL, "seqs, n_tokens or tokens is NULL");
  if (n_seqs <= 0) return fail(FS_ERR_EMPTY, "a batch needs at least one segment");
  fs_status s;
  if ((s = check_out_ptr(logits, "logits_out")) != FS_OK) return s;
  if ((s = check_i32_out(argmax, "argmax_out")) != FS_OK) return s;
  long long total = 0;
  const int cap = kv_capacity(kv);
  for (int i = 0; i < n_seqs; ++i) {
    const int q = seqs[i];
    if (q < 0 || q >= kv->max_seqs) return fail(FS_ERR_SEQ, "sequence out of range");
    for (int j = 0; j < i; ++j)
      if (seqs[j] == q) return fail(FS_ERR_SEQ, "a sequence appears twice in one batch");
    if (n_tokens[i] <= 0) return fail(FS_ERR_EMPTY, "every segment needs at least one token");
    if ((long long)kv->len[q] + n_tokens[i] > cap)
      return fail(FS_ERR_CONTEXT, "a segment would exceed max_pos or the KV capacity");
    total += n_tokens[i];
  }
  if (total > kMaxBatch) return fail(FS_ERR_INVALID, "a batch holds at most 64 rows in all");
  const int rows = (int)total;
  std::vector<int32_t> in(rows);
  if (pointer_kind(tokens) == 1) {
    FS_CUDA(cudaMemcpyAsync(in.data(), tokens, (size_t)rows * sizeof(int32_t),
                            cudaMemcpyDeviceToHost, st));
    FS_CUDA(cudaStreamSynchronize(st));
  } else {
    std::copy(tokens, tokens + rows, in.begin());
  }
  RowMap map{};
  map.n_list = rows;
  std::vector<int32_t> ordered(rows);
  int r = 0, c0 = 0;
  for (int i = 0; i < n_seqs; ++i) {  // all but the last row of every segment
    for (int t = 0; t + 1 < n_tokens[i]; ++t, ++r) {
      map.seq[r] = seqs[i];
      map.pos[r] = kv->len[seqs[i]] + t;
      ordered[r] = in[c0 + t];
    }
    c0 += n_tokens[i];
  }
  c0 = 0;
  for (int i = 0; i < n_seqs; ++i, ++r) {  // the last rows
    const int t = n_tokens[i] - 1;
    map.seq[r] = seqs[i];
    map.pos[r] = kv->len[seqs[i]] + t;
    ordered[r] = in[c0 + t];
    c0 += n_tokens[i];
  }
  const int32_t* dev_tok = nullptr;
  if ((s = stage_tokens(m, ordered.data(), rows, m->tok, &dev_tok, st)) != FS_OK) return s;
  if ((s = forward_general(m, kv, map, rows, dev_tok, rows - n_seqs, logits, argmax, 0, rows,
                           st)) != FS_OK)
    return s;
  for (int i = 0; i < n_seqs; ++i) kv->len[seqs[i]] += n_tokens[i];
  if (m->capture) m->capture = nullptr;
  return FS_OK;
}

}  // namespace fs

extern "C" fs_status fs_prefill(fs_model* m, fs_kv* kv, int32_t seq, const int32_t* tokens,
                                int32_t n, float* logits, int32_t* argmax, void* stream) {
  return fs::prefill_impl(m, kv, seq, tokens, n, logits, argmax,
                          static_cast<cudaStream_t>(stream));
}

extern "C" fs_status fs_forward_batch(fs_model* m, fs_kv* kv, const int32_t* seqs,
                                      const int32_t* n_tokens, int32_t n_seqs,
                                      const int32_t* tokens, float* logits, int32_t* argmax,
                                      void* stream) {
  return fs::batch_impl(m, kv, seqs, n_tokens, n_seqs, tokens, logits, argmax,
                        static_cast<cudaStream_t>(stream));
}

extern "C" fs_status fs_decode_step(fs_model* m, fs_kv* kv, const int32_t* seqs,
                                    const int32_t* tokens, int32_t batch, float* logits,
                                    int32_t* argmax, void* stream) {
  return fs::decode_impl(m, kv, seqs, tokens, batch, logits, argmax,
                         static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// Generation: greedy (fs_greedy) and seeded sampling (fs_generate)

namespace {

struct Sampler {
  float temperature;  // > 0 (greedy generation passes no sampler)
  int32_t top_k;
  float top_p;
  uint64_t seed;
};

fs_status check_sampler(float temperature, int32_t top_k, float top_p) {
  if (!(temperature >= 0.f) || !std::isfinite(temperature))
    return fail(FS_ERR_INVALID, "temperature must be finite and >= 0");
  if (top_k < 0) return fail(FS_ERR_INVALID, "top_k must be >= 0");
  if (!(top_p > 0.f && top_p <= 1.f)) return fail(FS_ERR_INVALID, "top_p must be in (0, 1]");
  return FS_OK;
}

// The next id from the last row's logits (lg, device fp32 [V]) into *dst:
// the sampler's draw for generated-token index `step`.
fs_status sample_into(fs_model* m, const Sampler& sp, const float* lg, uint64_t step, int32_t* dst,
                      cudaStream_t st) {
  FS_CUDA(fs::launch_sample(lg, 1, m->s.V, sp.temperature, sp.top_k, sp.top_p, sp.seed, step, dst,
                            st));
  return FS_OK;
}

// Prompt -> ids under the stop contract of "Coming back to Failed Star", "Next:
// one complete deterministic generation arc". Each forward's last-row logits
// give the next id: the greedy argmax (sp == nullptr) or the sampler's draw.
fs_status generate_impl(fs_model* m, fs_kv* kv, int32_t seq, const int32_t* prompt,
                        int32_t n_prompt, int32_t max_new, const int32_t* eos, int32_t n_eos,
                        const Sampler* sp, int32_t* out_tokens, int32_t* n_out,
                        int32_t* stop_reason, cudaStream_t st) {
  if (!m || !kv || !n_out || !stop_reason) return fail(FS_ERR_NULL, "NULL argument");
  if (kv->model != m) return fail(FS_ERR_INVALID, "kv belongs to another model");
  if (n_prompt <= 0) return fail(FS_ERR_EMPTY, "empty prompt");
  if (!prompt) return fail(FS_ERR_NULL, "prompt is NULL");
  if (max_new < 0) return fail(FS_ERR_INVALID, "max_new < 0");
  if (n_eos < 0 || (n_eos > 0 && !eos)) return fail(FS_ERR_INVALID, "bad EOS list");
  if (seq < 0 || seq >= kv->max_seqs) return fail(FS_ERR_SEQ, "sequence out of range");
  const int limit = fs::kv_capacity(kv);
  const int n = kv->len[seq] + n_prompt;
  if (n > limit) return fail(FS_ERR_CONTEXT, "prompt exceeds max_pos or the KV capacity");
  *n_out = 0;
  if (max_new == 0) {
    *stop_reason = FS_STOP_BUDGET;
    return FS_OK;
  }
  if (max_new > 0 && !out_tokens) return fail(FS_ERR_NULL, "out_tokens is NULL");
  // Forwards can run at prefix lengths n .. limit, one id each.
  const long long possible = (long long)limit - n + 1;
  const int steps = (int)std::min<long long>(max_new, possible);
  int reason = (max_new <= possible) ? FS_STOP_BUDGET : FS_STOP_CONTEXT;
  fs_status s = fs::ensure_gen_buffer(m, steps);
  if (s != FS_OK) return s;
  int32_t* gen = m->gen_tok;
  float* lg = sp ? m->lm_scratch : nullptr;
  if ((s = fs::prefill_impl(m, kv, seq, prompt, n_prompt, lg, sp ? nullptr : gen, st)) != FS_OK)
    return s;
  if (sp && (s = sample_into(m, *sp, lg, 0, gen, st)) != FS_OK) return s;
  const int base_len = kv->len[seq];  // == n
  std::vector<int32_t> host(steps);
  int produced = steps;
  const int chunk = n_eos > 0 ? 32 : steps;
  int done = 1;
  bool stopped = false;
  int checked = 0;
  while (!stopped) {
    const int upto = std::min(steps, std::max(done, 1) + (done == 1 ? chunk - 1 : chunk));
    for (int i = done; i < upto; ++i) {
      if ((s = fs::decode_impl(m, kv, &seq, gen + i - 1, 1, lg, sp ? nullptr : gen + i, st)) !=
          FS_OK)
        return s;
      if (sp && (s = sample_into(m, *sp, lg, (uint64_t)i, gen + i, st)) != FS_OK) return s;
    }
    done = upto;
    if (n_eos > 0) {
      FS_CUDA(cudaMemcpyAsync(host.data(), gen, (size_t)done * sizeof(int32_t),
                              cudaMemcpyDeviceToHost, st));
      FS_CUDA(cudaStreamSynchronize(st));
      for (int i = checked; i < done && !stopped; ++i)
        for (int e = 0; e < n_eos; ++e)
          if (host[i] == eos[e]) {
            produced = i + 1;
            reason = FS_STOP_EOS;
            stopped = true;
            break;
          }
      checked = done;
    }
    if (done >= steps) break;
  }
  // Forwards that ran past an EOS leave positions beyond the returned ids;
  // the sequence keeps exactly the positions its returned ids imply.
  kv->len[seq] = base_len + produced - 1;
  if (pointer_kind(out_tokens) == 1) {
    FS_CUDA(cudaMemcpyAsync(out_tokens, gen, (size_t)produced * sizeof(int32_t),
                            cudaMemcpyDeviceToDevice, st));
  } else {
    FS_CUDA(cudaMemcpyAsync(out_tokens, gen, (size_t)produced * sizeof(int32_t),
                            cudaMemcpyDeviceToHost, st));
  }
  FS_CUDA(cudaStreamSynchronize(st));
  int derr = 0;
  FS_CUDA(cudaMemcpy(&derr, m->err, sizeof(int), cudaMemcpyDeviceToHost));
  if (derr) {
    cudaMemset(m->err, 0, sizeof(int));
    fs::fused_reset(m);
    fs::cluster_reset(m);
    fs::mega_reset(m);
    return fail(FS_ERR_DEVICE, "a kernel reported device error " + std::to_string(derr));
  }
  *n_out = produced;
  *stop_reason = reason;
  return FS_OK;
}

}  // namespace

extern "C" fs_status fs_greedy(fs_model* m, fs_kv* kv, int32_t seq, const int32_t* prompt,
                               int32_t n_prompt, int32_t max_new, const int32_t* eos,
                               int32_t n_eos, int32_t* out_tokens, int32_t* n_out,
                               int32_t* stop_reason, void* stream) {
  return generate_impl(m, kv, seq, prompt, n_prompt, max_new, eos, n_eos, nullptr, out_tokens,
                       n_out, stop_reason, static_cast<cudaStream_t>(stream));
}

extern "C" fs_status fs_generate(fs_model* m, fs_kv* kv, int32_t seq, const int32_t* prompt,
                                 int32_t n_prompt, int32_t max_new, const int32_t* eos,
                                 int32_t n_eos, float temperature, int32_t top_k, float top_p,
                                 uint64_t seed, int32_t* out_tokens, int32_t* n_out,
                                 int32_t* stop_reason, void* stream) {
  fs_status s = check_sampler(temperature, top_k, top_p);
  if (s != FS_OK) return s;
  Sampler sp{temperature, top_k, top_p, seed};
  return generate_impl(m, kv, seq, prompt, n_prompt, max_new, eos, n_eos,
                       temperature > 0.f ? &sp : nullptr, out_tokens, n_out, stop_reason,
                       static_cast<cudaStream_t>(stream));
}

extern "C" fs_status fs_sample(fs_model* m, const float* logits, int32_t rows, float temperature,
                               int32_t top_k, float top_p, uint64_t seed, uint64_t step,
                               int32_t* out_ids, void* stream) {
  if (!m) return fail(FS_ERR_NULL, "model is NULL");
  if (rows <= 0 || rows > fs::kMaxBatch) return fail(FS_ERR_INVALID, "rows must be in [1, 64]");
  fs_status s = check_sampler(temperature, top_k, top_p);
  if (s != FS_OK) return s;
  if ((s = check_device_ptr(logits, "logits")) != FS_OK) return s;
  if (!out_ids) return fail(FS_ERR_NULL, "out_ids is NULL");
  if ((s = check_i32_out(out_ids, "out_ids")) != FS_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (temperature == 0.f) {
    FS_CUDA(fs::launch_argmax_rows(logits, rows, m->s.V, out_ids, st));
  } else {
    FS_CUDA(fs::launch_sample(logits, rows, m->s.V, temperature, top_k, top_p, seed, step, out_ids,
                              st));
  }
  return FS_OK;
}

// ---------------------------------------------------------------------------
// Debug entry points

extern "C" fs_status fs_debug_capture(fs_model* m, float* hidden, int32_t max_rows) {
  if (!m) return fail(FS_ERR_NULL, "model is NULL");
  if (!hidden) {
    m->capture = nullptr;
    return FS_OK;
  }
  fs_status s = check_device_ptr(hidden, "hidden");
  if (s != FS_OK) return s;
  if (max_rows <= 0) return fail(FS_ERR_INVALID, "max_rows must be positive");
  m->capture = hidden;
  m->capture_max_rows = max_rows;
  return FS_OK;
}

extern "C" fs_status fs_debug_block(fs_model* m, fs_kv* kv, int32_t seq, int32_t layer,
                                    const float* h_in, int32_t rows, float* h_out, void* stream) {
  if (!m || !kv) return fail(FS_ERR_NULL, "model or kv is NULL");
  if (kv->model != m) return fail(FS_ERR_INVALID, "kv belongs to another model");
  if (seq < 0 || seq >= kv->max_seqs) return fail(FS_ERR_SEQ, "sequence out of range");
  if (layer < 0 || layer >= m->s.L) return fail(FS_ERR_INVALID, "layer out of range");
  if (rows <= 0 || rows > m->max_rows) return fail(FS_ERR_INVALID, "rows out of range");
  fs_status s;
  if ((s = check_device_ptr(h_in, "h_in")) != FS_OK || (s = check_device_ptr(h_out, "h_out")) != FS_OK)
    return s;
  const int pos0 = kv->len[seq];
  if ((long long)pos0 + rows > fs::kv_capacity(kv))
    return fail(FS_ERR_CONTEXT, "block rows would exceed the KV capacity");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  fs::RowMap map{};
  map.n_list = 0;
  map.seq0 = seq;
  map.pos0 = pos0;
  if (rows == 1) {
    map.n_list = 1;
    map.seq[0] = seq;
    map.pos[0] = pos0;
    s = fs::decode_persistent(m, kv, map, 1, nullptr, h_in, h_out, layer, layer + 1, false, nullptr,
                         nullptr, st);
    if (s != FS_ERR_UNSUPPORTED) return s;
  }
  FS_CUDA(cudaMemcpyAsync(m->h, h_in, (size_t)rows * m->s.H * sizeof(float),
                          cudaMemcpyDeviceToDevice, st));
  if ((s = fs::block_prefill_or_general(m, kv, map, rows, layer, st)) != FS_OK) return s;
  FS_CUDA(cudaMemcpyAsync(h_out, m->h, (size_t)rows * m->s.H * sizeof(float),
                          cudaMemcpyDeviceToDevice, st));
  return FS_OK;
}

extern "C" fs_status fs_debug_dequant_q8_0(const int8_t* codes, const void* scales, int32_t n,
                                           int32_t k, float* out, void* stream) {
  if (n < 0 || k < 0 || k % 32) return fail(FS_ERR_INVALID, "need n >= 0 and k % 32 == 0");
  if ((size_t)n * k == 0) return FS_OK;
  fs_status s;
  if ((s = check_device_ptr(codes, "codes")) != FS_OK ||
      (s = check_device_ptr(scales, "scales")) != FS_OK ||
      (s = check_device_ptr(out, "out")) != FS_OK)
    return s;
  FS_CUDA(fs::launch_dequant_q8_0(codes, static_cast<const __half*>(scales), n, k, out,
                                  static_cast<cudaStream_t>(stream)));
  return FS_OK;
}

extern "C" fs_status fs_debug_lm_head(fs_model* m, const float* x, int32_t rows, float* logits,
                                      int32_t* argmax, void* stream) {
  if (!m) return fail(FS_ERR_NULL, "model is NULL");
  if (rows <= 0 || rows > fs::kMaxBatch) return fail(FS_ERR_INVALID, "rows must be in [1, 64]");
  fs_status s;
  if ((s = check_device_ptr(x, "x")) != FS_OK) return s;
  if ((s = check_out_ptr(logits, "logits")) != FS_OK) return s;
  if ((s = check_i32_out(argmax, "argmax")) != FS_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  FS_CUDA(fs::launch_rmsnorm(x, rows, m->s.H, m->final_norm, m->s.eps, m->xf, st));
  FS_CUDA(fs::launch_lm_head(m->xf, rows, m->s, m->embed, logits, argmax, m->partial, m->n_part,
                             m->err, st));
  return FS_OK;
}

extern "C" fs_status fs_debug_wait_limit(fs_model* m, uint64_t wait_ns, int32_t withhold_layer) {
  if (!m) return fail(FS_ERR_NULL, "model is NULL");
  if (wait_ns < 1000 || wait_ns > 60000000000ull)
    return fail(FS_ERR_INVALID, "wait limit must be in [1 us, 60 s]");
  if (withhold_layer < -1 || withhold_layer >= m->s.L)
    return fail(FS_ERR_INVALID, "withhold_layer must be -1 or a layer index");
  fs::fused_debug_wait(m, wait_ns, withhold_layer);
  fs::cluster_debug_wait(m, wait_ns, withhold_layer);
  fs::mega_debug_wait(m, wait_ns, withhold_layer);
  return FS_OK;
}

extern "C" fs_status fs_debug_decode_path(fs_model* m, int32_t path) {
  if (!m) return fail(FS_ERR_NULL, "model is NULL");
  if (path < 0 || path > 4) return fail(FS_ERR_INVALID, "path must be 0 .. 4");
  m->decode_path = path;
  return FS_OK;
}

extern "C" fs_status fs_debug_decode_kernel(const fs_model* m, int32_t batch, int32_t* kind) {
  if (!m || !kind) return fail(FS_ERR_NULL, "model or kind is NULL");
  if (batch < 1 || batch > fs::kMaxBatch) return fail(FS_ERR_INVALID, "batch out of range");
  *kind = 0;
  const int path = m->decode_path;
  if (batch > 4 || path == 2) return FS_OK;
  if ((path == 3 || (path == 0 && batch == 1)) && fs::mega_eligible(m)) {
    *kind = 3;
  } else if (path == 3) {
    *kind = 0;
  } else if ((path == 0 || path == 4) && fs::cluster_eligible(m)) {
    *kind = 2;
  } else {
    *kind = path == 4 ? 0 : 1;
  }
  return FS_OK;
}

extern "C" fs_status fs_debug_trace(fs_model* m, uint64_t* buf) {
  if (!m) return fail(FS_ERR_NULL, "model is NULL");
  if (buf) {
    fs_status s = check_device_ptr(buf, "trace buffer");
    if (s != FS_OK) return s;
  }
  m->trace = reinterpret_cast<unsigned long long*>(buf);
  return FS_OK;
}

extern "C" const char* fs_last_error_string(void) { return g_last_error.c_str(); }

extern "C" const char* fs_status_string(fs_status s) {
  switch (s) {
    case FS_OK: return "FS_OK";
    case FS_ERR_INVALID: return "FS_ERR_INVALID";
    case FS_ERR_NULL: return "FS_ERR_NULL";
    case FS_ERR_ALIGN: return "FS_ERR_ALIGN";
    case FS_ERR_OOM: return "FS_ERR_OOM";
    case FS_ERR_EMPTY: return "FS_ERR_EMPTY";
    case FS_ERR_TOKEN: return "FS_ERR_TOKEN";
    case FS_ERR_CONTEXT: return "FS_ERR_CONTEXT";
    case FS_ERR_CUDA: return "FS_ERR_CUDA";
    case FS_ERR_SEQ: return "FS_ERR_SEQ";
    case FS_ERR_DEVICE: return "FS_ERR_DEVICE";
    case FS_ERR_UNSUPPORTED: return "FS_ERR_UNSUPPORTED";
    default: return "unknown fs_status";
  }
}
