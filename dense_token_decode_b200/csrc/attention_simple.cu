// Causal GQA attention over the paged bf16 KV cache, one CTA per (row, query
// head), CUDA cores, online softmax in fp32. Row r at position p attends keys
// 0..p of its sequence; query head h reads kv head h / (nq / nkv). It takes
// what the specialised kernels do not cover (any row count, any position mix,
// head sizes or GQA groups outside their templates).
#include "fs_internal.h"

namespace fs {

namespace {

template <int E>  // E = head_dim / 32 elements per lane
__global__ void __launch_bounds__(128) attention_simple_kernel(const float* __restrict__ q,
                                                               const RowMap map, int nq,
                                                               int nkv, KVView kv, int layer,
                                                               float* __restrict__ o) {
  constexpr int d = 32 * E;
  __shared__ float sm_m[4], sm_l[4];
  __shared__ float sm_acc[4][d];
  const int r = blockIdx.x, h = blockIdx.y;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = h / (nq / nkv);
  const RowInfo ri = map.get(r);
  const float scale = 1.f / sqrtf((float)d);
  float qv[E], acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    qv[e] = q[((size_t)r * nq + h) * d + lane * E + e];
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int j = w; j <= ri.pos; j += 4) {
    const size_t off = kv.offset(layer, ri.seq, j, g) + lane * E;
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) s = fmaf(qv[e], __bfloat162float(kv.k[off + e]), s);
    for (int x = 16; x > 0; x >>= 1) s += __shfl_xor_sync(0xffffffffu, s, x);
    s *= scale;
    const float mn = fmaxf(m, s);
    const float corr = expf(m - mn), p = expf(s - mn);
    l = l * corr + p;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = acc[e] * corr + p * __bfloat162float(kv.v[off + e]);
    m = mn;
  }
  if (lane == 0) {
    sm_m[w] = m;
    sm_l[w] = l;
  }
#pragma unroll
  for (int e = 0; e < E; ++e) sm_acc[w][lane * E + e] = acc[e];
  __syncthreads();
  if (w == 0) {
    float M = sm_m[0];
    for (int i = 1; i < 4; ++i) M = fmaxf(M, sm_m[i]);
    float L = 0.f, f[4];
    for (int i = 0; i < 4; ++i) {
      f[i] = (sm_m[i] == -INFINITY) ? 0.f : expf(sm_m[i] - M);
      L += sm_l[i] * f[i];
    }
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int c = lane * E + e;
      float v = 0.f;
      for (int i = 0; i < 4; ++i) v += sm_acc[i][c] * f[i];
      o[((size_t)r * nq + h) * d + c] = v / L;
    }
  }
}

}  // namespace

cudaError_t launch_attention_simple(const float* q, int rows, const RowMap& map,
                                    const Shape& s, KVView kv, int layer, float* o,
                                    cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  dim3 grid(rows, s.nq);
  if (s.d != 128 && s.d != 64) return cudaErrorInvalidValue;
  count_launches();
  if (s.d == 128)
    attention_simple_kernel<4><<<grid, 128, 0, st>>>(q, map, s.nq, s.nkv, kv, layer, o);
  else
    attention_simple_kernel<2><<<grid, 128, 0, st>>>(q, map, s.nq, s.nkv, kv, layer, o);
  return cudaGetLastError();
}

}  // namespace fs
