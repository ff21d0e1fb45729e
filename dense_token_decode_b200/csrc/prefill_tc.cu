// Prefill blocks on the tensor cores: the state the tcgen05 GEMMs need (fp16
// copies of the weights, fp16 activation operands, TMA descriptors) and the
// per-block kernel sequence
//   RMSNorm -> fp16 operand (two terms when split) -> QKV GEMM whose epilogue
//   does the q/k head norm + RoPE + KV append -> tensor-core attention (fp16 out)
//   -> O GEMM (+= residual) -> RMSNorm -> fp16 operand
//   -> gate/up GEMM with SwiGLU epilogue (fp16 act) -> down GEMM (+= residual).
#include <cuda.h>

#include <vector>

#include "runtime.h"
#include "tc_common.cuh"

namespace fs {

cudaError_t launch_gemm_tc(const CUtensorMap* a, const CUtensorMap* a_lo, const CUtensorMap* b,
                           const CUtensorMap* b2, int M, int N, int K, int kind, float* out,
                           int ldo, __half* act_hi, __half* act_lo, int act_ld, int* err,
                           int num_sms, cudaStream_t st, int bn, int lo_col0 = 0);
cudaError_t launch_gemm_tc_qkv_heads(const CUtensorMap* a, const CUtensorMap* a_lo,
                                     const CUtensorMap* b, int M, int N, int K, int* err,
                                     int num_sms, cudaStream_t st, int bn, int lo_col0,
                                     const float2* rope, const __nv_bfloat16* q_norm,
                                     const __nv_bfloat16* k_norm, float eps, int nq, int nkv,
                                     int d, const KVView& kv, int layer, int seq, int pos0,
                                     float* q_out);

namespace {

// ---------------------------------------------------------------------------
// Small kernels

__global__ void bf16_to_f16_kernel(const __nv_bfloat16* __restrict__ src, size_t n,
                                   __half* __restrict__ dst) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    dst[i] = __float2half_rn(__bfloat162float(src[i]));
}

__global__ void q8_to_f16_kernel(const int8_t* __restrict__ codes, const __half* __restrict__ sc,
                                 size_t n, int k, __half* __restrict__ dst) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t r = i / k, c = i % k;
    dst[i] = __float2half_rn((float)codes[i] * __half2float(sc[r * (k / 32) + c / 32]));
  }
}

// RMSNorm of fp32 rows into fp16 operand terms: hi = fp16(y), lo = fp16(y - hi).
__global__ void __launch_bounds__(256) rmsnorm_f16_kernel(const float* __restrict__ x, int H,
                                                          const __nv_bfloat16* __restrict__ g,
                                                          float eps, __half* __restrict__ hi,
                                                          __half* __restrict__ lo) {
  pdl_trigger();
  pdl_wait();
  __shared__ float red[8];
  const float* xr = x + (size_t)blockIdx.x * H;
  float ss = 0.f;
  for (int c = threadIdx.x; c < H; c += 256) ss += xr[c] * xr[c];
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float t = 0.f;
  for (int w = 0; w < 8; ++w) t += red[w];
  const float inv = rsqrtf(t / (float)H + eps);
  for (int c = threadIdx.x; c < H; c += 256) {
    const float y = xr[c] * inv * __bfloat162float(g[c]);
    const __half h = __float2half_rn(y);
    hi[(size_t)blockIdx.x * H + c] = h;
    if (lo) lo[(size_t)blockIdx.x * H + c] = __float2half_rn(y - __half2float(h));
  }
}

__global__ void f32_to_f16_kernel(const float* __restrict__ x, size_t n, __half* __restrict__ hi) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    hi[i] = __float2half_rn(x[i]);
}

int grid_for(size_t n) {
  const size_t b = (n + 255) / 256;
  return (int)(b < 8192 ? b : 8192);
}

struct LayerMaps {
  CUtensorMap qkv, o, g, u, d;
};

struct TcState {
  bool ready = false;
  bool failed = false;
  __half* w16 = nullptr;  // per layer: qkv [qkvd,H] | o [H,qd] | g [I,H] | u [I,H] | d [H,I]
  __half *xn_hi = nullptr, *xn_lo = nullptr, *o_hi = nullptr, *act_hi = nullptr;
  std::vector<LayerMaps> maps;
  CUtensorMap a_xn_hi, a_xn_lo, a_o, a_act;
};

}  // namespace

static TcState* tc_state(fs_model* m) {
  return static_cast<TcState*>(m->tc_extras);
}

void tc_release(fs_model* m) {
  TcState* t = tc_state(m);
  if (!t) return;
  void* bufs[] = {t->w16, t->xn_hi, t->xn_lo, t->o_hi, t->act_hi};
  for (void* b : bufs)
    if (b) cudaFree(b);
  delete t;
  m->tc_extras = nullptr;
}

// Output tile widths: 256 where the output is wide (fewer re-reads of the
// activations per FLOP), 128 for the H-wide outputs (enough tiles for the SMs).
static int bn_qkv(const Shape& s) { return s.qkv_dim() % 256 == 0 ? 256 : 128; }
static int bn_gu(const Shape& s) { return s.I % 128 == 0 ? 256 : 128; }

// Whether the tensor-core prefill covers this model's shape.
static bool tc_shape_ok(const fs_model* m) {
  const Shape& s = m->s;
  return s.H % 128 == 0 && s.q_dim() % 128 == 0 && s.qkv_dim() % 128 == 0 && s.I % 64 == 0 &&
         s.H % 64 == 0 && s.I % 64 == 0 && s.q_dim() % 64 == 0;
}

// Builds the fp16 weight copies and operand buffers on first use.
static fs_status tc_prepare(fs_model* m, cudaStream_t st) {
  TcState* t = tc_state(m);
  if (t && t->ready) return FS_OK;
  if (t && t->failed) return FS_ERR_UNSUPPORTED;
  if (!tc_shape_ok(m)) return FS_ERR_UNSUPPORTED;
  if (!t) {
    t = new TcState();
    m->tc_extras = t;
  }
  const Shape& s = m->s;
  const size_t R = m->max_rows;
  const size_t per_layer = (size_t)s.qkv_dim() * s.H + (size_t)s.H * s.q_dim() +
                           2 * (size_t)s.I * s.H + (size_t)s.H * s.I;
  auto fail = [&](fs_status code, const char* what) {
    t->failed = true;
    set_error(what);
    return code;
  };
  if (cudaMalloc(&t->w16, per_layer * s.L * sizeof(__half)) != cudaSuccess ||
      cudaMalloc(&t->xn_hi, R * s.H * sizeof(__half)) != cudaSuccess ||
      cudaMalloc(&t->xn_lo, R * s.H * sizeof(__half)) != cudaSuccess ||
      cudaMalloc(&t->o_hi, R * s.q_dim() * sizeof(__half)) != cudaSuccess ||
      cudaMalloc(&t->act_hi, R * s.I * sizeof(__half)) != cudaSuccess) {
    cudaGetLastError();
    return fail(FS_ERR_OOM, "out of device memory for the fp16 prefill weights");
  }
  t->maps.resize(s.L);
  for (int l = 0; l < s.L; ++l) {
    const LayerDev& Lw = m->layers[l];
    __half* base = t->w16 + per_layer * l;
    __half* wqkv = base;
    __half* wo = wqkv + (size_t)s.qkv_dim() * s.H;
    __half* wg = wo + (size_t)s.H * s.q_dim();
    __half* wu = wg + (size_t)s.I * s.H;
    __half* wd = wu + (size_t)s.I * s.H;
    struct Part {
      int which;
      __half* dst;
      int n, k;
    } parts[7] = {{kWq, wqkv, s.q_dim(), s.H},
                  {kWk, wqkv + (size_t)s.q_dim() * s.H, s.kv_dim(), s.H},
                  {kWv, wqkv + (size_t)(s.q_dim() + s.kv_dim()) * s.H, s.kv_dim(), s.H},
                  {kWo, wo, s.H, s.q_dim()},
                  {kWg, wg, s.I, s.H},
                  {kWu, wu, s.I, s.H},
                  {kWd, wd, s.H, s.I}};
    for (const Part& pt : parts) {
      const size_t n = (size_t)pt.n * pt.k;
      count_launches();
      if (m->q8)
        q8_to_f16_kernel<<<grid_for(n), 256, 0, st>>>(static_cast<const int8_t*>(Lw.w[pt.which]),
                                                      Lw.s[pt.which], n, pt.k, pt.dst);
      else
        bf16_to_f16_kernel<<<grid_for(n), 256, 0, st>>>(
            static_cast<const __nv_bfloat16*>(Lw.w[pt.which]), n, pt.dst);
    }
    LayerMaps& mp = t->maps[l];
    if (!make_tmap_16(&mp.qkv, wqkv, s.qkv_dim(), s.H, bn_qkv(s), false) ||
        !make_tmap_16(&mp.o, wo, s.H, s.q_dim(), 128, false) ||
        !make_tmap_16(&mp.g, wg, s.I, s.H, bn_gu(s) / 2, false) ||
        !make_tmap_16(&mp.u, wu, s.I, s.H, bn_gu(s) / 2, false) ||
        !make_tmap_16(&mp.d, wd, s.H, s.I, 128, false))
      return fail(FS_ERR_UNSUPPORTED, "the driver refused a TMA descriptor");
  }
  if (!make_tmap_16(&t->a_xn_hi, t->xn_hi, (int)R, s.H, 128, false) ||
      !make_tmap_16(&t->a_xn_lo, t->xn_lo, (int)R, s.H, 128, false) ||
      !make_tmap_16(&t->a_o, t->o_hi, (int)R, s.q_dim(), 128, false) ||
      !make_tmap_16(&t->a_act, t->act_hi, (int)R, s.I, 128, false))
    return fail(FS_ERR_UNSUPPORTED, "the driver refused a TMA descriptor");
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(FS_ERR_CUDA, "fp16 weight conversion failed");
  t->ready = true;
  return FS_OK;
}

bool attention_tc_supported(const Shape& s, const KVView& kv, const RowMap& map);
cudaError_t launch_attention_tc(const float* q, int rows, const RowMap& map, const Shape& s,
                                const KVView& kv, int layer, __half* o, int* err,
                                cudaStream_t st);

bool tc_available(fs_model* m, cudaStream_t st) { return tc_prepare(m, st) == FS_OK; }

// One block on the tensor cores over m->h (rows >= 1; the M tail is masked).
fs_status layer_tc(fs_model* m, const fs_kv* kv, const RowMap& map, int rows, int l,
                   cudaStream_t st) {
  TcState* t = tc_state(m);
  const Shape& s = m->s;
  const LayerDev& Lw = m->layers[l];
  const LayerMaps& mp = t->maps[l];
  const KVView kvv = kv_view(kv);
  const bool split = m->prefill_split != 0;
  // The second operand term matters where the output is rounded to bf16 in
  // the cache (the K and V columns); the Q columns use one fp16 term.
  const int split_from = s.q_dim() % bn_qkv(s) == 0 ? s.q_dim() : 0;
  cudaError_t e;
#define FS_TRY(x)                                                     \
  do {                                                                \
    e = (x);                                                          \
    if (e != cudaSuccess) {                                           \
      set_error(std::string("prefill block: ") + cudaGetErrorString(e)); \
      return FS_ERR_CUDA;                                             \
    }                                                                 \
  } while (0)
  count_launches();
  FS_TRY(launch_pdl(rmsnorm_f16_kernel, dim3(rows), dim3(256), 0, st, (const float*)m->h, s.H,
                    (const __nv_bfloat16*)Lw.attn_norm, s.eps, t->xn_hi,
                    split ? t->xn_lo : (__half*)nullptr));
  if (map.n_list == 0 && bn_qkv(s) % s.d == 0 && s.d % 64 == 0) {
    // the per-head RMSNorm, RoPE and the K/V append run in the GEMM epilogue
    FS_TRY(launch_gemm_tc_qkv_heads(&t->a_xn_hi, split ? &t->a_xn_lo : nullptr, &mp.qkv, rows,
                                    s.qkv_dim(), s.H, m->err, m->num_sms, st, bn_qkv(s),
                                    split_from, m->rope, Lw.q_norm, Lw.k_norm, s.eps, s.nq,
                                    s.nkv, s.d, kvv, l, map.seq0, map.pos0, m->q));
  } else {
    FS_TRY(launch_gemm_tc(&t->a_xn_hi, split ? &t->a_xn_lo : nullptr, &mp.qkv, nullptr, rows,
                          s.qkv_dim(), s.H, 0, m->qkv, s.qkv_dim(), nullptr, nullptr, 0, m->err,
                          m->num_sms, st, bn_qkv(s), split_from));
    FS_TRY(launch_qk_norm_rope_append(m->qkv, rows, map, s, Lw.q_norm, Lw.k_norm, m->rope, m->q,
                                      kvv, l, st));
  }
  if (attention_tc_supported(s, kvv, map)) {
    FS_TRY(launch_attention_tc(m->q, rows, map, s, kvv, l, t->o_hi, m->err, st));
  } else {
    FS_TRY(launch_attention_simple(m->q, rows, map, s, kvv, l, m->o, st));
    const size_t no = (size_t)rows * s.q_dim();
    count_launches();
    f32_to_f16_kernel<<<grid_for(no), 256, 0, st>>>(m->o, no, t->o_hi);
    FS_TRY(cudaGetLastError());
  }
  FS_TRY(launch_gemm_tc(&t->a_o, nullptr, &mp.o, nullptr, rows, s.H, s.q_dim(), 1, m->h, s.H,
                        nullptr, nullptr, 0, m->err, m->num_sms, st, 128));
  count_launches();
  FS_TRY(launch_pdl(rmsnorm_f16_kernel, dim3(rows), dim3(256), 0, st, (const float*)m->h, s.H,
                    (const __nv_bfloat16*)Lw.ffn_norm, s.eps, t->xn_hi, (__half*)nullptr));
  FS_TRY(launch_gemm_tc(&t->a_xn_hi, nullptr, &mp.g, &mp.u, rows, 2 * s.I, s.H, 2, nullptr, 0,
                        t->act_hi, nullptr, s.I, m->err, m->num_sms, st, bn_gu(s)));
  FS_TRY(launch_gemm_tc(&t->a_act, nullptr, &mp.d, nullptr, rows, s.H, s.I, 1, m->h, s.H, nullptr,
                        nullptr, 0, m->err, m->num_sms, st, 128));
#undef FS_TRY
  return FS_OK;
}

}  // namespace fs
