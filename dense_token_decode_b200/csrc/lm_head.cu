// Tied LM head with greedy selection for a few rows: logits[r, v] =
// sum_k xf[r, k] E[v, k] with xf the final-RMSNormed row, then the argmax
// over the finite logits with the lowest id winning an exact tie ("Coming
// back to Failed Star", "Next: one complete deterministic generation arc",
// Selection). Stage 1 streams E once (warp per vocab row, 16-byte loads) and
// keeps each CTA's best (value, id) per row; stage 2 reduces the CTA partials.
#include "fs_internal.h"

namespace fs {

namespace {

__device__ __forceinline__ float lo16(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float hi16(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// (value, id) order of the greedy choice: larger value wins, equal values go
// to the lower id; non-finite values never win.
__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

template <int R>
__global__ void __launch_bounds__(256) lm_head_kernel(const float* __restrict__ xf, int rows,
                                                      int H, int V,
                                                      const __nv_bfloat16* __restrict__ E,
                                                      float* __restrict__ logits,
                                                      float2* __restrict__ partial) {
  __shared__ float sv[8][R];
  __shared__ int si[8][R];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float bv[R];
  int bi[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    bv[r] = -INFINITY;
    bi[r] = 0x7fffffff;
  }
  const int chunks = H / 8;
  for (int v = blockIdx.x * 8 + w; v < V; v += gridDim.x * 8) {
    const uint4* er = reinterpret_cast<const uint4*>(E + (size_t)v * H);
    float acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0.f;
#pragma unroll 4
    for (int c = lane; c < chunks; c += 32) {
      const uint4 e = __ldg(er + c);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (r >= rows) break;
        const float4 a = *reinterpret_cast<const float4*>(xf + (size_t)r * H + c * 8);
        const float4 b = *reinterpret_cast<const float4*>(xf + (size_t)r * H + c * 8 + 4);
        float s = acc[r];
        s = fmaf(lo16(e.x), a.x, s);
        s = fmaf(hi16(e.x), a.y, s);
        s = fmaf(lo16(e.y), a.z, s);
        s = fmaf(hi16(e.y), a.w, s);
        s = fmaf(lo16(e.z), b.x, s);
        s = fmaf(hi16(e.z), b.y, s);
        s = fmaf(lo16(e.w), b.z, s);
        s = fmaf(hi16(e.w), b.w, s);
        acc[r] = s;
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (r >= rows) break;
      float s = acc[r];
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) {
        if (logits) logits[(size_t)r * V + v] = s;
        if (isfinite(s) && better(s, v, bv[r], bi[r])) {
          bv[r] = s;
          bi[r] = v;
        }
      }
    }
  }
  if (lane == 0) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      sv[w][r] = bv[r];
      si[w][r] = bi[r];
    }
  }
  __syncthreads();
  if (threadIdx.x < R && threadIdx.x < rows) {
    const int r = threadIdx.x;
    float v = sv[0][r];
    int i = si[0][r];
    for (int k = 1; k < 8; ++k)
      if (better(sv[k][r], si[k][r], v, i)) {
        v = sv[k][r];
        i = si[k][r];
      }
    partial[(size_t)r * gridDim.x + blockIdx.x] = make_float2(v, __int_as_float(i));
  }
}

__global__ void argmax_final_kernel(const float2* __restrict__ partial, int n_part,
                                    int32_t* __restrict__ argmax, int* err) {
  __shared__ float sv[32];
  __shared__ int si[32];
  const int r = blockIdx.x;
  float v = -INFINITY;
  int i = 0x7fffffff;
  for (int k = threadIdx.x; k < n_part; k += blockDim.x) {
    const float2 p = partial[(size_t)r * n_part + k];
    const int pi = __float_as_int(p.y);
    if (better(p.x, pi, v, i)) {
      v = p.x;
      i = pi;
    }
  }
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, v, o);
    const int oi = __shfl_xor_sync(0xffffffffu, i, o);
    if (better(ov, oi, v, i)) {
      v = ov;
      i = oi;
    }
  }
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    sv[w] = v;
    si[w] = i;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int k = 1; k < (int)(blockDim.x >> 5); ++k)
      if (better(sv[k], si[k], v, i)) {
        v = sv[k];
        i = si[k];
      }
    if (i == 0x7fffffff) {  // no finite logit
      i = 0;
      if (err) atomicCAS(err, 0, kErrBounds);
    }
    argmax[r] = i;
  }
}

}  // namespace

cudaError_t launch_lm_head(const float* x, int rows, const Shape& s, const __nv_bfloat16* E,
                           float* logits, int32_t* argmax, float2* partial, int n_part, int* err,
                           cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  for (int r0 = 0; r0 < rows; r0 += 16) {
    const int rr = rows - r0 < 16 ? rows - r0 : 16;
    const float* xr = x + (size_t)r0 * s.H;
    float* lr = logits ? logits + (size_t)r0 * s.V : nullptr;
    float2* pr = partial + (size_t)r0 * n_part;
#define FS_LM_CASE(RR)                                                                    \
  if (rr <= RR) {                                                                         \
    count_launches();                                                                     \
    lm_head_kernel<RR><<<n_part, 256, 0, st>>>(xr, rr, s.H, s.V, E, lr, pr);              \
  } else
    FS_LM_CASE(1) FS_LM_CASE(2) FS_LM_CASE(4) FS_LM_CASE(8) FS_LM_CASE(16) {}
#undef FS_LM_CASE
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (argmax) {
      count_launches();
      argmax_final_kernel<<<rr, 256, 0, st>>>(pr, n_part, argmax + r0, err);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
  }
  return cudaSuccess;
}

}  // namespace fs
