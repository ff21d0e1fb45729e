// Weight-streaming linear layer for 5..16 rows (batched decode, bf16
// weights): y[r, n] (+)= sum_k x[r, k] W[n, k].
//
// One warp owns 8 weight rows and a 256-wide slice of the input axis: every
// lane loads 8 consecutive bf16 weights of each of the 8 rows (16-byte loads,
// 512 contiguous bytes per row per warp) and the matching 8 activations of
// each batch row, so an activation load serves 8 weight rows and a weight
// load serves every batch row. The 8 x R partial sums are reduced across the
// warp by a transposing butterfly (4 sums per lane at the end) and added
// into y with fp32 atomics, which combine the slices of the input axis.
// Many short warps keep enough weight bytes in flight to stream HBM.
#include "fs_internal.h"

namespace fs {

namespace {

constexpr int kRowsPerWarp = 8;
constexpr int kSlice = 256;  // input-axis slice of one warp
constexpr int kWarps = 4;

__device__ __forceinline__ float lo16(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float hi16(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// Transposing butterfly over the warp: 128 partial sums per lane in, the
// warp totals of 4 of them per lane out. Rounds with masks 16, 8, 4, 2, 1
// halve the values a lane keeps (64, 32, 16, 8, 4); afterwards lane l holds
// in v[q] the total of index 64*b4 + 32*b3 + 16*b2 + 8*b1 + 4*b0 + q, with
// b4..b0 the bits of l.
__device__ __forceinline__ void reduce128(float (&v)[128], int lane) {
#pragma unroll
  for (int w = 64, mask = 16; w >= 4; w >>= 1, mask >>= 1) {
    const bool upper = (lane & mask) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float send = upper ? v[i] : v[i + w];
      const float keep = upper ? v[i + w] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
    }
  }
}

template <int R>
__global__ void __launch_bounds__(kWarps * 32) gemv_splitk_kernel(
    const float* __restrict__ x, int rows, int K, const __nv_bfloat16* __restrict__ W, int N,
    float* __restrict__ out, int ldo) {
  const int lane = threadIdx.x & 31;
  const int gw = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int slices = K / kSlice;
  const int n_groups = (N + kRowsPerWarp - 1) / kRowsPerWarp;
  if (gw >= n_groups * slices) return;
  const int grp = gw / slices, sl = gw % slices;
  const int n0 = grp * kRowsPerWarp;
  const int k = sl * kSlice + lane * 8;

  uint4 w[kRowsPerWarp];
#pragma unroll
  for (int j = 0; j < kRowsPerWarp; ++j) {
    const int n = min(n0 + j, N - 1);  // rows past N repeat the last one; dropped below
    w[j] = __ldg(reinterpret_cast<const uint4*>(W + (size_t)n * K + k));
  }
  float v[128];
#pragma unroll
  for (int i = 0; i < 128; ++i) v[i] = 0.f;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (r >= rows) break;
    const float4 a = __ldg(reinterpret_cast<const float4*>(x + (size_t)r * K + k));
    const float4 b = __ldg(reinterpret_cast<const float4*>(x + (size_t)r * K + k + 4));
#pragma unroll
    for (int j = 0; j < kRowsPerWarp; ++j) {
      float s = lo16(w[j].x) * a.x;
      s = fmaf(hi16(w[j].x), a.y, s);
      s = fmaf(lo16(w[j].y), a.z, s);
      s = fmaf(hi16(w[j].y), a.w, s);
      s = fmaf(lo16(w[j].z), b.x, s);
      s = fmaf(hi16(w[j].z), b.y, s);
      s = fmaf(lo16(w[j].w), b.z, s);
      s = fmaf(hi16(w[j].w), b.w, s);
      v[r * 8 + j] = s;
    }
  }
  reduce128(v, lane);
  const int base = ((lane >> 4) & 1) * 64 + ((lane >> 3) & 1) * 32 + ((lane >> 2) & 1) * 16 +
                   ((lane >> 1) & 1) * 8 + (lane & 1) * 4;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int idx = base + q, r = idx >> 3, j = idx & 7;
    if (r < rows && n0 + j < N) atomicAdd(out + (size_t)r * ldo + n0 + j, v[q]);
  }
}

// Greedy choice per row over finite logits, the lowest id winning an exact
// tie (the same rule as the LM-head kernels). One CTA per row.
__global__ void __launch_bounds__(1024) argmax_rows_kernel(const float* __restrict__ logits,
                                                           int V, int32_t* __restrict__ argmax) {
  __shared__ float sv[32];
  __shared__ int si[32];
  const float* row = logits + (size_t)blockIdx.x * V;
  float bv = -INFINITY;
  int bi = 0x7fffffff;
  for (int v = threadIdx.x; v < V; v += blockDim.x) {
    const float x = row[v];
    if (isfinite(x) && (x > bv || (x == bv && v < bi))) {
      bv = x;
      bi = v;
    }
  }
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ov > bv || (ov == bv && oi < bi)) {
      bv = ov;
      bi = oi;
    }
  }
  if ((threadIdx.x & 31) == 0) {
    sv[threadIdx.x >> 5] = bv;
    si[threadIdx.x >> 5] = bi;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int nw = blockDim.x >> 5;
    bv = threadIdx.x < nw ? sv[threadIdx.x] : -INFINITY;
    bi = threadIdx.x < nw ? si[threadIdx.x] : 0x7fffffff;
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (threadIdx.x == 0) argmax[blockIdx.x] = bi == 0x7fffffff ? 0 : bi;
  }
}

}  // namespace

cudaError_t launch_argmax_rows(const float* logits, int rows, int V, int32_t* argmax,
                               cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  count_launches();
  argmax_rows_kernel<<<rows, 1024, 0, st>>>(logits, V, argmax);
  return cudaGetLastError();
}

bool gemv_splitk_ok(int rows, int K, const __half* scales) {
  return scales == nullptr && rows >= 1 && rows <= 16 && K % kSlice == 0;
}

// y (+)= x W^T over `rows` rows; out rows are ldo floats apart. Without
// `accumulate` the output block is cleared first.
cudaError_t launch_gemv_splitk(const float* x, int rows, int K, const __nv_bfloat16* W, int N,
                               float* out, int ldo, bool accumulate, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  if (!accumulate) {
    cudaError_t e = cudaMemset2DAsync(out, (size_t)ldo * sizeof(float), 0, (size_t)N * sizeof(float),
                                      rows, st);
    if (e != cudaSuccess) return e;
  }
  const int warps = (N + kRowsPerWarp - 1) / kRowsPerWarp * (K / kSlice);
  const int blocks = (warps + kWarps - 1) / kWarps;
  count_launches();
  gemv_splitk_kernel<16><<<blocks, kWarps * 32, 0, st>>>(x, rows, K, W, N, out, ldo);
  return cudaGetLastError();
}

}  // namespace fs
