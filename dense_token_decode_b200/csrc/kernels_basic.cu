// Row-wise kernels of the forward pass: embedding lookup, RMSNorm, SwiGLU,
// the per-head q/k RMSNorm + RoPE + KV-cache append, Q8_0 dequantisation and
// KV import/export. They are small next to the weight streaming and serve the
// general (any row count) path.
#include "fs_internal.h"

namespace fs {

__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

__device__ __forceinline__ void set_err(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

template <int NW>
__device__ __forceinline__ float block_sum(float v, float* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = (l < NW) ? red[l] : 0.f;
  for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  __syncthreads();
  return t;
}

// ---------------------------------------------------------------------------
// Embedding: h[r, :] = E[tokens[r], :] widened to fp32 ("Coming back to Failed
// Star", data-flow figure: ids[S] -> embedding[S,H]).
__global__ void embed_kernel(const int32_t* __restrict__ tokens,
                             const __nv_bfloat16* __restrict__ E, int H, int V,
                             float* __restrict__ h, int* err) {
  const int r = blockIdx.x;
  int t = tokens[r];
  if (t < 0 || t >= V) {
    if (threadIdx.x == 0) set_err(err, kErrToken);
    t = 0;
  }
  const uint4* src = reinterpret_cast<const uint4*>(E + (size_t)t * H);
  float4* dst = reinterpret_cast<float4*>(h + (size_t)r * H);
  for (int c = threadIdx.x; c < H / 8; c += blockDim.x) {
    const uint4 u = __ldg(src + c);
    dst[2 * c] = make_float4(bf16lo(u.x), bf16hi(u.x), bf16lo(u.y), bf16hi(u.y));
    dst[2 * c + 1] = make_float4(bf16lo(u.z), bf16hi(u.z), bf16lo(u.w), bf16hi(u.w));
  }
}

cudaError_t launch_embed(const int32_t* tokens, int rows, const __nv_bfloat16* E, int H, int V,
                         float* h, int* err, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  count_launches();
  embed_kernel<<<rows, 128, 0, st>>>(tokens, E, H, V, h, err);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// RMSNorm of each row: out = x / sqrt(mean(x^2) + eps) * g, fp32. With
// `zero`, row r also clears zero_w floats at zero + r * zero_ld (the output
// block of the accumulating product that reads `out` next).
__global__ void __launch_bounds__(256) rmsnorm_kernel(const float* __restrict__ x, int H,
                                                      const __nv_bfloat16* __restrict__ g,
                                                      float eps, float* __restrict__ out,
                                                      float* __restrict__ zero, int zero_w,
                                                      int zero_ld) {
  __shared__ float red[8];
  pdl_trigger();
  pdl_wait();
  if (zero)
    for (int c = threadIdx.x; c < zero_w; c += 256) zero[(size_t)blockIdx.x * zero_ld + c] = 0.f;
  const float4* xr = reinterpret_cast<const float4*>(x + (size_t)blockIdx.x * H);
  float ss = 0.f;
  for (int c = threadIdx.x; c < H / 4; c += 256) {
    const float4 v = xr[c];
    ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  ss = block_sum<8>(ss, red);
  const float inv = rsqrtf(ss / (float)H + eps);
  float4* o = reinterpret_cast<float4*>(out + (size_t)blockIdx.x * H);
  const uint2* gp = reinterpret_cast<const uint2*>(g);
  for (int c = threadIdx.x; c < H / 4; c += 256) {
    const float4 v = xr[c];
    const uint2 gg = __ldg(gp + c);
    o[c] = make_float4(v.x * inv * bf16lo(gg.x), v.y * inv * bf16hi(gg.x),
                       v.z * inv * bf16lo(gg.y), v.w * inv * bf16hi(gg.y));
  }
}

cudaError_t launch_rmsnorm(const float* x, int rows, int H, const __nv_bfloat16* g, float eps,
                           float* out, cudaStream_t st, float* zero, int zero_w, int zero_ld) {
  if (rows <= 0) return cudaSuccess;
  count_launches();
  return launch_pdl(rmsnorm_kernel, dim3(rows), dim3(256), 0, st, x, H, g, eps, out, zero, zero_w,
                    zero_ld);
}

// ---------------------------------------------------------------------------
// SwiGLU on a [rows, 2I] gate||up buffer: act = silu(gate) * up.
__global__ void swiglu_kernel(const float* __restrict__ gu, int rows, int I,
                              float* __restrict__ act) {
  const size_t n = (size_t)rows * I;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t r = i / I, j = i % I;
    const float g = gu[r * 2 * I + j], u = gu[r * 2 * I + I + j];
    act[i] = g / (1.f + expf(-g)) * u;
  }
}

cudaError_t launch_swiglu(const float* gu, int rows, int I, float* act, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  const size_t n = (size_t)rows * I;
  const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  count_launches();
  swiglu_kernel<<<blocks, 256, 0, st>>>(gu, rows, I, act);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Per-head q/k RMSNorm over head_dim, rotate-half RoPE at the row's position,
// and the KV append. One warp per head: warps [0, nq) take the query heads,
// warps [nq, nq+nkv) take one kv head each (K normalised and rotated, V as
// is), both rounded to bf16 into the sequence's page. qkv rows are
// [q (nq*d) | k (nkv*d) | v (nkv*d)] fp32.
// Lane layout: with E = d/64 elements per lane per half, lane l owns
// elements l*E+e of the first half and d/2 + l*E+e of the second half, so a
// rotation pair (i, i+d/2) sits in one lane.
template <int E>
__global__ void qk_norm_rope_append_kernel(const float* __restrict__ qkv, const RowMap map,
                                           int nq, int nkv, float eps,
                                           const __nv_bfloat16* __restrict__ q_norm,
                                           const __nv_bfloat16* __restrict__ k_norm,
                                           const float2* __restrict__ rope,
                                           float* __restrict__ q_out, KVView kv, int layer) {
  pdl_trigger();
  pdl_wait();
  constexpr int d = 64 * E, half = 32 * E;
  const int r = blockIdx.x, w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qkv_dim = (nq + 2 * nkv) * d;
  const RowInfo ri = map.get(r);
  const float* row = qkv + (size_t)r * qkv_dim;
  const bool is_q = w < nq;
  const int head = is_q ? w : w - nq;
  const float* src = is_q ? row + head * d : row + nq * d + head * d;
  const __nv_bfloat16* gain = is_q ? q_norm : k_norm;
  float lo[E], hi[E];
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    lo[e] = src[lane * E + e];
    hi[e] = src[half + lane * E + e];
    ss += lo[e] * lo[e] + hi[e] * hi[e];
  }
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = rsqrtf(ss / (float)d + eps);
  const float2* cs = rope + (size_t)ri.pos * half;
  float olo[E], ohi[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = lane * E + e;
    const float a = lo[e] * inv * __bfloat162float(gain[i]);
    const float b = hi[e] * inv * __bfloat162float(gain[half + i]);
    const float2 t = cs[i];
    olo[e] = a * t.x - b * t.y;
    ohi[e] = b * t.x + a * t.y;
  }
  if (is_q) {
    float* dst = q_out + (size_t)r * nq * d + head * d;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      dst[lane * E + e] = olo[e];
      dst[half + lane * E + e] = ohi[e];
    }
  } else {
    const size_t off = kv.offset(layer, ri.seq, ri.pos, head);
    const float* vsrc = row + nq * d + nkv * d + head * d;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      kv.k[off + lane * E + e] = __float2bfloat16_rn(olo[e]);
      kv.k[off + half + lane * E + e] = __float2bfloat16_rn(ohi[e]);
      kv.v[off + lane * E + e] = __float2bfloat16_rn(vsrc[lane * E + e]);
      kv.v[off + half + lane * E + e] = __float2bfloat16_rn(vsrc[half + lane * E + e]);
    }
  }
}

cudaError_t launch_qk_norm_rope_append(const float* qkv, int rows, const RowMap& map,
                                       const Shape& s, const __nv_bfloat16* q_norm,
                                       const __nv_bfloat16* k_norm, const float2* rope,
                                       float* q_out, KVView kv, int layer, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  const int threads = 32 * (s.nq + s.nkv);
  if (s.d != 128 && s.d != 64) return cudaErrorInvalidValue;
  count_launches();
  if (s.d == 128)
    return launch_pdl(qk_norm_rope_append_kernel<2>, dim3(rows), dim3(threads), 0, st, qkv, map,
                      s.nq, s.nkv, s.eps, q_norm, k_norm, rope, q_out, kv, layer);
  return launch_pdl(qk_norm_rope_append_kernel<1>, dim3(rows), dim3(threads), 0, st, qkv, map, s.nq,
                    s.nkv, s.eps, q_norm, k_norm, rope, q_out, kv, layer);
}

// ---------------------------------------------------------------------------
// Q8_0 dequantisation (debug / bit-exactness check): w = q * s exactly.
__global__ void dequant_q8_0_kernel(const int8_t* __restrict__ codes,
                                    const __half* __restrict__ scales, size_t total, int k,
                                    float* __restrict__ out) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t n = i / k, c = i % k;
    out[i] = (float)codes[i] * __half2float(scales[n * (k / 32) + c / 32]);
  }
}

cudaError_t launch_dequant_q8_0(const int8_t* codes, const __half* scales, int n, int k,
                                float* out, cudaStream_t st) {
  const size_t total = (size_t)n * k;
  if (!total) return cudaSuccess;
  const int blocks = (int)((total + 255) / 256 < 8192 ? (total + 255) / 256 : 8192);
  count_launches();
  dequant_q8_0_kernel<<<blocks, 256, 0, st>>>(codes, scales, total, k, out);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// KV import/export between a logical [n, nkv, d] array and the pages of one
// (sequence, layer). 16-byte chunks.
__global__ void kv_copy_kernel(KVView kv, int seq, int layer, int pos0, int n,
                               __nv_bfloat16* k, __nv_bfloat16* v, bool import) {
  const int cpr = kv.head_dim / 8;  // chunks per head row
  const size_t total = (size_t)n * kv.n_kv_heads * cpr;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const int c = (int)(i % cpr);
    const int g = (int)((i / cpr) % kv.n_kv_heads);
    const int t = (int)(i / ((size_t)cpr * kv.n_kv_heads));
    const size_t off = kv.offset(layer, seq, pos0 + t, g) + c * 8;
    uint4* pk = reinterpret_cast<uint4*>(kv.k + off);
    uint4* pv = reinterpret_cast<uint4*>(kv.v + off);
    uint4* lk = reinterpret_cast<uint4*>(k) + i;
    uint4* lv = reinterpret_cast<uint4*>(v) + i;
    if (import) {
      *pk = *lk;
      *pv = *lv;
    } else {
      *lk = *pk;
      *lv = *pv;
    }
  }
}

cudaError_t launch_kv_copy(KVView kv, int seq, int layer, int pos0, int n, __nv_bfloat16* k,
                           __nv_bfloat16* v, bool import, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const size_t total = (size_t)n * kv.n_kv_heads * (kv.head_dim / 8);
  const int blocks = (int)((total + 255) / 256 < 8192 ? (total + 255) / 256 : 8192);
  count_launches();
  kv_copy_kernel<<<blocks, 256, 0, st>>>(kv, seq, layer, pos0, n, k, v, import);
  return cudaGetLastError();
}

}  // namespace fs
