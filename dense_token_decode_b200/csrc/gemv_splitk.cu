// Weight-streaming linear layer for 5..16 rows (batched decode, bf16
// weights): y[r, n] (+)= sum_k x[r, k] W[n, k], on the tensor cores.
//
// mma.sync m16n8k16 (bf16 in, fp32 accumulate) with the batch rows as M (16,
// rows past `rows` zero) and 8 weight rows as N. A CTA takes one 256-wide
// slice of the input axis: it stages the slice of x once in shared memory as
// two bf16 terms (hi and the lo remainder, about 16 significant bits), and
// its 8 warps each stream tasks of 8 weight rows of it straight from global
// memory into registers (16-byte loads); a warp runs `tpw` tasks (more than
// one only for very wide outputs, to share the staged slice). The k order inside an MMA is a fixed
// permutation of the physical k: lane (g, t) holds weights 8t .. 8t + 7 of
// a 32-wide group, used as the B pairs (8t, 8t + 1 | 8t + 2, 8t + 3) of one
// MMA and (8t + 4, .. | 8t + 6, ..) of the next, and the A fragments of x
// are read with the same mapping, so every product pairs matching k. The
// accumulators need no shuffles: each lane adds its 4 outputs into y with
// fp32 atomics, which combine the slices of the input axis.
#include "fs_internal.h"

namespace fs {

namespace {

constexpr int kSlice = 256;        // input-axis slice of a CTA
constexpr int kWarps = 8;
constexpr int kRowsPerWarp = 8;    // weight rows of a warp task (one n8 tile)
constexpr int kXStride = kSlice + 32;  // bf16 per staged row (64-byte pad: no bank conflicts)

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Up to three products of the same input in one launch (q, k, v; gate, up):
// segment i multiplies x by W[i] (N[i] rows) into out[i]. Tasks of 8 weight
// rows are numbered across the segments.
struct Segs {
  const __nv_bfloat16* W[3];
  float* out[3];
  int N[3];
  int tasks[3];  // cumulative task counts
  int n;
};

// With `swiglu`, x rows are [gate (K) | up (K)] and the staged input is
// silu(gate) * up (the same expression as swiglu_kernel).
__global__ void __launch_bounds__(kWarps * 32) gemv_mma_kernel(
    const float* __restrict__ x, int rows, int K, const Segs sg, int ldo, int ctas_per_slice,
    int tpw, int swiglu) {
  // [term][16 rows][kXStride] bf16
  __shared__ __align__(16) __nv_bfloat16 xs[2][16][kXStride];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int slice = blockIdx.x / ctas_per_slice, cs = blockIdx.x % ctas_per_slice;
  const int k0 = slice * kSlice;
  const int g = lane >> 2, t = lane & 3;
  const int n_tasks = sg.tasks[sg.n - 1];
  // The first task's weights are requested before the slice of x is staged,
  // so the HBM latency overlaps the staging. Weights: row n0 + g, 8 groups of
  // 32 k; lane t holds 8t .. 8t + 7 of each.
  uint4 w[8];
  int seg = 0, n0 = 0;
  auto load_w = [&](int task) {
    seg = task < sg.tasks[0] ? 0 : (task < sg.tasks[1] ? 1 : 2);
    n0 = (task - (seg ? sg.tasks[seg - 1] : 0)) * kRowsPerWarp;
    const int N = sg.N[seg];
    const int n = min(n0 + g, N - 1);  // rows past N repeat the last one; dropped below
    const __nv_bfloat16* wr = sg.W[seg] + (size_t)n * K + k0 + 8 * t;
#pragma unroll
    for (int q = 0; q < 8; ++q) w[q] = __ldg(reinterpret_cast<const uint4*>(wr + 32 * q));
  };
  int task = cs * tpw * kWarps + warp;
  if (task < n_tasks) load_w(task);
  // everything below reads or writes what earlier kernels wrote or read
  pdl_trigger();
  pdl_wait();
  for (int e = tid; e < 16 * kSlice; e += kWarps * 32) {
    const int r = e / kSlice, c = e % kSlice;
    float v = 0.f;
    if (r < rows) {
      if (swiglu) {
        const float gt = x[(size_t)r * 2 * K + k0 + c], up = x[(size_t)r * 2 * K + K + k0 + c];
        v = gt / (1.f + expf(-gt)) * up;
      } else {
        v = x[(size_t)r * K + k0 + c];
      }
    }
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    xs[0][r][c] = h;
    xs[1][r][c] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
  __syncthreads();
  for (int it = 0; it < tpw; ++it, task += kWarps) {
    if (task >= n_tasks) break;
    if (it > 0) load_w(task);
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};  // hi, lo chains
#pragma unroll
    for (int q = 0; q < 8; ++q) {
#pragma unroll
      for (int term = 0; term < 2; ++term) {
        const uint4 xa = *reinterpret_cast<const uint4*>(&xs[term][g][32 * q + 8 * t]);
        const uint4 xb = *reinterpret_cast<const uint4*>(&xs[term][g + 8][32 * q + 8 * t]);
        mma_bf16(acc[term], xa.x, xb.x, xa.y, xb.y, w[q].x, w[q].y);
        mma_bf16(acc[term], xa.z, xb.z, xa.w, xb.w, w[q].z, w[q].w);
      }
    }
    // D[batch row][weight row]: (g, 2t), (g, 2t + 1), (g + 8, 2t), (g + 8, 2t + 1)
    float* out = sg.out[seg];
    const int N = sg.N[seg];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int r = g + (e >> 1) * 8, n = n0 + 2 * t + (e & 1);
      if (r < rows && n < N) atomicAdd(out + (size_t)r * ldo + n, acc[0][e] + acc[1][e]);
    }
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

namespace {

cudaError_t launch_segs(const float* x, int rows, int K, Segs sg, int ldo, cudaStream_t st,
                        int swiglu = 0) {
  const int n_tasks = sg.tasks[sg.n - 1];
  const int slices = K / kSlice;
  // one task per warp unless the grid would exceed ~4 waves of 3 CTAs per SM
  int tpw = 1;
  while (tpw < 8 && (long long)n_tasks * slices / (kWarps * tpw) > 148LL * 3 * 4) tpw *= 2;
  const int ctas_per_slice = (n_tasks + kWarps * tpw - 1) / (kWarps * tpw);
  const int blocks = ctas_per_slice * slices;
  count_launches();
  return launch_pdl(gemv_mma_kernel, dim3(blocks), dim3(kWarps * 32), 0, st, x, rows, K, sg, ldo,
                    ctas_per_slice, tpw, swiglu);
}

}  // namespace

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
  Segs sg{};
  sg.W[0] = W;
  sg.out[0] = out;
  sg.N[0] = N;
  sg.tasks[0] = (N + kRowsPerWarp - 1) / kRowsPerWarp;
  sg.n = 1;
  return launch_segs(x, rows, K, sg, ldo, st);
}

// Products of one input with n (2 or 3) matrices, written side by side: W[i]
// (N[i] rows) into columns out0 + sum_{j<i} N[j] of rows ldo floats apart,
// which are cleared first unless the caller has (`cleared`).
cudaError_t launch_gemv_splitk_multi(const float* x, int rows, int K, int n,
                                     const __nv_bfloat16* const* W, const int* N, float* out0,
                                     int ldo, bool cleared, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  if (n < 1 || n > 3) return cudaErrorInvalidValue;
  int width = 0;
  for (int i = 0; i < n; ++i) width += N[i];
  if (!cleared) {
    cudaError_t e = cudaMemset2DAsync(out0, (size_t)ldo * sizeof(float), 0,
                                      (size_t)width * sizeof(float), rows, st);
    if (e != cudaSuccess) return e;
  }
  Segs sg{};
  int col = 0, tasks = 0;
  for (int i = 0; i < n; ++i) {
    sg.W[i] = W[i];
    sg.out[i] = out0 + col;
    sg.N[i] = N[i];
    tasks += (N[i] + kRowsPerWarp - 1) / kRowsPerWarp;
    sg.tasks[i] = tasks;
    col += N[i];
  }
  for (int i = n; i < 3; ++i) sg.tasks[i] = tasks;
  sg.n = n;
  return launch_segs(x, rows, K, sg, ldo, st);
}

// y += silu(gate) * up times W^T over `rows` rows (accumulating into out).
cudaError_t launch_gemv_splitk_swiglu(const float* gu, int rows, int K, const __nv_bfloat16* W,
                                      int N, float* out, int ldo, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  Segs sg{};
  sg.W[0] = W;
  sg.out[0] = out;
  sg.N[0] = N;
  sg.tasks[0] = (N + kRowsPerWarp - 1) / kRowsPerWarp;
  sg.n = 1;
  return launch_segs(gu, rows, K, sg, ldo, st, 1);
}

}  // namespace fs
