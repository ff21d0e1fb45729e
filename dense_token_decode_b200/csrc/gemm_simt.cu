// Plain shared-memory tiled GEMM on the CUDA cores (fp32 arithmetic):
// C[m, n] (+)= sum_k A[m, k] W[n, k], A fp32 [M, K], W bf16 or Q8_0 [N, K].
// It serves the general path for 17..127 rows (decode batches above 16, short
// prefill chunks) and shapes the tensor-core GEMM does not cover; it makes no
// attempt at peak throughput.
#include "fs_internal.h"

namespace fs {

namespace {

constexpr int BM = 64, BN = 64, BK = 32;

template <bool Q8>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const float* __restrict__ A, int M, int K,
                                                        const void* __restrict__ W,
                                                        const __half* __restrict__ scales, int N,
                                                        float* __restrict__ C, int ldc,
                                                        bool accumulate) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Ws[BK][BN + 4];
  const int tid = threadIdx.x;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int tm = (tid / 16) * 4, tn = (tid % 16) * 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += BK) {
    // 64x32 tiles of A and W, 8 elements per thread each.
    for (int i = tid; i < BM * BK; i += 256) {
      const int r = i / BK, c = i % BK;
      const int m = m0 + r, n = n0 + r, k = k0 + c;
      As[c][r] = (m < M) ? A[(size_t)m * K + k] : 0.f;
      float w = 0.f;
      if (n < N) {
        if (Q8)
          w = (float)static_cast<const int8_t*>(W)[(size_t)n * K + k] *
              __half2float(scales[(size_t)n * (K / 32) + k / 32]);
        else
          w = __bfloat162float(static_cast<const __nv_bfloat16*>(W)[(size_t)n * K + k]);
      }
      Ws[c][r] = w;
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < BK; ++c) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[c][tm + i];
        b[i] = Ws[c][tn + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + tm + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tn + j;
      if (n >= N) continue;
      float* p = C + (size_t)m * ldc + n;
      *p = accumulate ? *p + acc[i][j] : acc[i][j];
    }
  }
}

}  // namespace

cudaError_t launch_gemm_simt(const float* A, int M, int K, const void* W, const __half* scales,
                             int N, float* C, int ldc, bool accumulate, cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  if (K % BK) return cudaErrorInvalidValue;
  dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM);
  count_launches();
  if (scales)
    gemm_simt_kernel<true><<<grid, 256, 0, st>>>(A, M, K, W, scales, N, C, ldc, accumulate);
  else
    gemm_simt_kernel<false><<<grid, 256, 0, st>>>(A, M, K, W, scales, N, C, ldc, accumulate);
  return cudaGetLastError();
}

}  // namespace fs
