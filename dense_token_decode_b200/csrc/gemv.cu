// Weight-streaming GEMV for a few rows (decode): y[r, n] = sum_k x[r, k] W[n, k].
// W is bf16 [N, K] or Q8_0 (int8 codes [N, K] + fp16 scales [N, K/32]);
// x and y are fp32. One warp owns one output column n at a time and walks
// the contiguous weight row with 16-byte loads; the activations come through
// L1. The Q8_0 codes are widened and scaled in registers (w = q * s, exact in
// fp32), so only 1.0625 bytes per weight leave HBM.
#include "fs_internal.h"

namespace fs {

namespace {

__device__ __forceinline__ float lo16(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float hi16(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// 8 bf16 weights (one uint4) dotted with x[k0 .. k0+8).
__device__ __forceinline__ float dot8_bf16(const uint4 w, const float* x) {
  const float4 a = *reinterpret_cast<const float4*>(x);
  const float4 b = *reinterpret_cast<const float4*>(x + 4);
  float s = lo16(w.x) * a.x;
  s = fmaf(hi16(w.x), a.y, s);
  s = fmaf(lo16(w.y), a.z, s);
  s = fmaf(hi16(w.y), a.w, s);
  s = fmaf(lo16(w.z), b.x, s);
  s = fmaf(hi16(w.z), b.y, s);
  s = fmaf(lo16(w.w), b.z, s);
  s = fmaf(hi16(w.w), b.w, s);
  return s;
}

// 16 int8 codes (one uint4) dotted with x[k0 .. k0+16), times the block scale.
__device__ __forceinline__ float dot16_q8(const uint4 w, const float* x, float scale) {
  const uint32_t v[4] = {w.x, w.y, w.z, w.w};
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float4 a = *reinterpret_cast<const float4*>(x + 4 * j);
    s = fmaf((float)(int8_t)(v[j] & 0xff), a.x, s);
    s = fmaf((float)(int8_t)((v[j] >> 8) & 0xff), a.y, s);
    s = fmaf((float)(int8_t)((v[j] >> 16) & 0xff), a.z, s);
    s = fmaf((float)(int8_t)(v[j] >> 24), a.w, s);
  }
  return s * scale;
}

// Dot products of one weight row with R activation rows, summed over the warp.
template <int R, bool Q8>
__device__ __forceinline__ void warp_row_dot(const void* W, const __half* scales, int n, int K,
                                             const float* x, int rows, float acc[R]) {
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = 0.f;
  const int lane = threadIdx.x & 31;
  if (!Q8) {
    const uint4* wr = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(W) +
                                                     (size_t)n * K);
    const int chunks = K / 8;
#pragma unroll 4
    for (int c = lane; c < chunks; c += 32) {
      const uint4 w = __ldg(wr + c);
#pragma unroll
      for (int r = 0; r < R; ++r)
        if (r < rows) acc[r] += dot8_bf16(w, x + (size_t)r * K + c * 8);
    }
  } else {
    const uint4* wr =
        reinterpret_cast<const uint4*>(static_cast<const int8_t*>(W) + (size_t)n * K);
    const __half* sr = scales + (size_t)n * (K / 32);
    const int chunks = K / 16;
#pragma unroll 4
    for (int c = lane; c < chunks; c += 32) {
      const uint4 w = __ldg(wr + c);
      const float sc = __half2float(sr[c >> 1]);
#pragma unroll
      for (int r = 0; r < R; ++r)
        if (r < rows) acc[r] += dot16_q8(w, x + (size_t)r * K + c * 16, sc);
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r)
    for (int o = 16; o > 0; o >>= 1) acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], o);
}

template <int R, bool Q8>
__global__ void __launch_bounds__(256) gemv_kernel(const float* __restrict__ x, int rows, int K,
                                                   const void* __restrict__ W,
                                                   const __half* __restrict__ scales, int N,
                                                   float* __restrict__ out, int ldo,
                                                   bool accumulate) {
  const int warps = gridDim.x * 8;
  for (int n = blockIdx.x * 8 + (threadIdx.x >> 5); n < N; n += warps) {
    float acc[R];
    warp_row_dot<R, Q8>(W, scales, n, K, x, rows, acc);
    if ((threadIdx.x & 31) == 0) {
#pragma unroll
      for (int r = 0; r < R; ++r)
        if (r < rows) {
          float* p = out + (size_t)r * ldo + n;
          *p = accumulate ? *p + acc[r] : acc[r];
        }
    }
  }
}

template <int R, bool Q8>
__global__ void __launch_bounds__(256) gemv_swiglu_kernel(
    const float* __restrict__ x, int rows, int K, const void* __restrict__ Wg,
    const __half* __restrict__ sg, const void* __restrict__ Wu, const __half* __restrict__ su,
    int N, float* __restrict__ act) {
  const int warps = gridDim.x * 8;
  for (int n = blockIdx.x * 8 + (threadIdx.x >> 5); n < N; n += warps) {
    float g[R], u[R];
    warp_row_dot<R, Q8>(Wg, sg, n, K, x, rows, g);
    warp_row_dot<R, Q8>(Wu, su, n, K, x, rows, u);
    if ((threadIdx.x & 31) == 0) {
#pragma unroll
      for (int r = 0; r < R; ++r)
        if (r < rows) act[(size_t)r * N + n] = g[r] / (1.f + expf(-g[r])) * u[r];
    }
  }
}

int gemv_blocks(int N) {
  int b = (N + 7) / 8;
  return b < 148 * 8 ? b : 148 * 8;
}

template <bool Q8>
cudaError_t gemv_dispatch(const float* x, int rows, int K, const void* W, const __half* s, int N,
                          float* out, int ldo, bool acc, cudaStream_t st) {
  const int b = gemv_blocks(N);
#define FS_GEMV_CASE(RR)                                                              \
  if (rows <= RR) {                                                                   \
    count_launches();                                                                 \
    gemv_kernel<RR, Q8><<<b, 256, 0, st>>>(x, rows, K, W, s, N, out, ldo, acc);       \
    return cudaGetLastError();                                                        \
  }
  FS_GEMV_CASE(1)
  FS_GEMV_CASE(2)
  FS_GEMV_CASE(4)
  FS_GEMV_CASE(8)
  FS_GEMV_CASE(16)
#undef FS_GEMV_CASE
  return cudaErrorInvalidValue;
}

template <bool Q8>
cudaError_t gemv_swiglu_dispatch(const float* x, int rows, int K, const void* Wg, const __half* sg,
                                 const void* Wu, const __half* su, int N, float* act,
                                 cudaStream_t st) {
  const int b = gemv_blocks(N);
#define FS_GEMV_CASE(RR)                                                                   \
  if (rows <= RR) {                                                                        \
    count_launches();                                                                      \
    gemv_swiglu_kernel<RR, Q8><<<b, 256, 0, st>>>(x, rows, K, Wg, sg, Wu, su, N, act);     \
    return cudaGetLastError();                                                             \
  }
  FS_GEMV_CASE(1)
  FS_GEMV_CASE(2)
  FS_GEMV_CASE(4)
  FS_GEMV_CASE(8)
  FS_GEMV_CASE(16)
#undef FS_GEMV_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_gemv(const float* x, int rows, int K, const void* W, const __half* scales,
                        int N, float* out, int ldo, bool accumulate, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  return scales ? gemv_dispatch<true>(x, rows, K, W, scales, N, out, ldo, accumulate, st)
                : gemv_dispatch<false>(x, rows, K, W, scales, N, out, ldo, accumulate, st);
}

cudaError_t launch_gemv_swiglu(const float* x, int rows, int K, const void* Wg, const __half* sg,
                               const void* Wu, const __half* su, int N, float* act,
                               cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  return sg ? gemv_swiglu_dispatch<true>(x, rows, K, Wg, sg, Wu, su, N, act, st)
            : gemv_swiglu_dispatch<false>(x, rows, K, Wg, sg, Wu, su, N, act, st);
}

}  // namespace fs
