// Weight-streaming linear layer for 5..16 rows (batched decode, bf16
// weights): y[r, n] (+)= sum_k x[r, k] W[n, k], on the tensor cores.
//
// A CTA (4 warps) owns 64 weight rows and a 256-column slice of the input
// axis (many CTAs per SM keep HBM busy). It stages the slice of every batch
// row in shared
// memory as two bf16 terms (hi = bf16(x), lo = bf16(x - hi)), so each product
// keeps about 16 bits of the fp32 activation; rows 2r and 2r + 1 of the
// operand hold the terms of batch row r. Each warp then streams its 16
// weight rows straight from global memory: per 32-column block a thread
// loads 8 consecutive weights of rows g and g + 8 (g = lane / 4, at column
// 32 blk + 8 (lane % 4)) and the same 8 columns of operand rows, an order of
// the columns that both operands share, and issues mma.sync m16n8k16 (bf16
// in, fp32 accumulate) for the four 8-column tiles of the 32 operand rows.
// The first weight loads are issued before the staging, and loads run
// several blocks ahead of the products. Slices of the input axis are
// combined with fp32 atomics.
#include "fs_internal.h"

namespace fs {

namespace {

constexpr int kWarps = 4;
constexpr int kRowsPerCta = 16 * kWarps;
constexpr int kSlice = 256;   // input-axis slice of one CTA
constexpr int kOpStride = kSlice + 8;  // bf16 per operand row in shared memory
constexpr int kAhead = 4;     // 32-column blocks of weights in flight per thread

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4],
                                         const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__global__ void __launch_bounds__(kWarps * 32) gemv_mma_kernel(
    const float* __restrict__ x, int rows, int K, const __nv_bfloat16* __restrict__ W, int N,
    float* __restrict__ out, int ldo) {
  extern __shared__ __align__(16) unsigned char smem[];
  __nv_bfloat16* op = reinterpret_cast<__nv_bfloat16*>(smem);  // [32][kOpStride]
  const int k0 = blockIdx.y * kSlice, ks = min(kSlice, K - k0);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, q = lane & 3;
  const int n0 = blockIdx.x * kRowsPerCta + warp * 16;
  const int ra = min(n0 + g, N - 1), rb = min(n0 + g + 8, N - 1);  // rows past N: dropped below
  const uint4* wa = reinterpret_cast<const uint4*>(W + (size_t)ra * K + k0 + 8 * q);
  const uint4* wb = reinterpret_cast<const uint4*>(W + (size_t)rb * K + k0 + 8 * q);
  const int nblk = ks / 32;
  uint4 pa[kAhead], pb[kAhead];
#pragma unroll
  for (int i = 0; i < kAhead; ++i) {
    pa[i] = i < nblk ? __ldg(wa + i * 4) : make_uint4(0u, 0u, 0u, 0u);
    pb[i] = i < nblk ? __ldg(wb + i * 4) : make_uint4(0u, 0u, 0u, 0u);
  }
  // stage the operand: 32 rows (hi, lo of 16 batch rows; absent rows zero)
  for (int i = threadIdx.x; i < 16 * ks; i += blockDim.x) {
    const int r = i / ks, k = i - r * ks;
    const float v = r < rows ? x[(size_t)r * K + k0 + k] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    op[(2 * r) * kOpStride + k] = hi;
    op[(2 * r + 1) * kOpStride + k] = __float2bfloat16_rn(v - __bfloat162float(hi));
  }
  __syncthreads();
  if (n0 >= N) return;
  const uint32_t opb = (uint32_t)__cvta_generic_to_shared(op) + (uint32_t)(g * kOpStride + 8 * q) * 2;
  float acc[4][4];
#pragma unroll
  for (int t = 0; t < 4; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[t][e] = 0.f;
  for (int blk0 = 0; blk0 < nblk; blk0 += kAhead) {
#pragma unroll
    for (int i = 0; i < kAhead; ++i) {
      const int blk = blk0 + i;
      if (blk >= nblk) break;
      const uint4 a = pa[i], b = pb[i];
      if (blk + kAhead < nblk) {
        pa[i] = __ldg(wa + (blk + kAhead) * 4);
        pb[i] = __ldg(wb + (blk + kAhead) * 4);
      }
      // k-step 0 takes columns 8q .. 8q+3 of the block, k-step 1 8q+4 .. 8q+7
      const uint32_t a0[4] = {a.x, b.x, a.y, b.y}, a1[4] = {a.z, b.z, a.w, b.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        uint4 z;
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(z.x), "=r"(z.y), "=r"(z.z), "=r"(z.w)
                     : "r"(opb + (uint32_t)(t * 8 * kOpStride + blk * 32) * 2));
        const uint32_t b0[2] = {z.x, z.y}, b1[2] = {z.z, z.w};
        mma16816(acc[t], a0, b0);
        mma16816(acc[t], a1, b1);
      }
    }
  }
  // acc[t]: rows g (e 0, 1) and g + 8 (e 2, 3) of the warp's 16, operand
  // columns 8t + 2q (hi) and 8t + 2q + 1 (lo): batch row 4t + q
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int r = 4 * t + q;
    if (r >= rows) continue;
    if (n0 + g < N) atomicAdd(out + (size_t)r * ldo + n0 + g, acc[t][0] + acc[t][1]);
    if (n0 + g + 8 < N) atomicAdd(out + (size_t)r * ldo + n0 + g + 8, acc[t][2] + acc[t][3]);
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
  return scales == nullptr && rows >= 1 && rows <= 16 && K % 32 == 0;
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
  static bool attr = false;
  const int smem = 32 * kOpStride * 2;
  if (!attr) {
    cudaFuncSetAttribute(gemv_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    attr = true;
  }
  const dim3 grid((N + kRowsPerCta - 1) / kRowsPerCta, (K + kSlice - 1) / kSlice);
  count_launches();
  gemv_mma_kernel<<<grid, kWarps * 32, smem, st>>>(x, rows, K, W, N, out, ldo);
  return cudaGetLastError();
}

}  // namespace fs
