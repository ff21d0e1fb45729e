// Tensor-core GEMM of the prefill path on sm_100a (tcgen05 + TMEM + TMA):
//   D[m, n] = sum_k A[m, k] * B[n, k]
// A: activations fp16 [M, K] (optionally two fp16 terms, A = A_hi + A_lo),
// B: weights fp16 [N, K] (the model's fp16 copy), both K-contiguous.
// Tiles of 128 (M) x 128 (N) with 64-wide K blocks; fp32 accumulators live in
// tensor memory, two buffers, so the epilogue of one tile runs while the
// next tile's MMAs are issued.
//
// Warp roles in a CTA of 192 threads (one CTA per SM, persistent over tiles):
//   warp 0: TMA producer (one lane) — A (and A_lo) and B blocks into a ring of
//           shared-memory stages with 128-byte swizzle;
//   warp 1: allocates TMEM, then one lane issues tcgen05.mma (M=128, N=128,
//           K=16 per instruction) and tcgen05.commit to release stages and
//           to hand finished accumulators to the epilogue;
//   warps 2-5: epilogue — tcgen05.ld of their 32 TMEM lanes (= tile rows),
//           then the fused output step of the GEMM kind.
//
// Every wait is bounded (%globaltimer); a timeout sets the error word and the
// CTA drains and frees TMEM before it returns.
#include <algorithm>

#include "runtime.h"
#include "tc_common.cuh"

namespace fs {
namespace tc {

constexpr int BM = 128, BK = 64;
constexpr int kThreads = 192;
constexpr int kTileBytes = BM * BK * 2;  // 16 KB for a 128 x 64 fp16 A tile

enum Kind { kStore = 0, kResidual = 1, kSwiGLU = 2, kQKVHead = 3 };

// kQKVHead epilogue: the QKV projection of consecutive positions pos0 + m of
// one sequence, finished per head in the epilogue: q and k heads RMSNorm'ed
// (gains over the head) and rotated (rotate-half RoPE at the row's position);
// q written fp32 [M][nq * d], k and v rounded to bf16 into the paged cache.
struct HeadEpi {
  const float2* rope;  // [max_pos][d/2] (cos, sin)
  const __nv_bfloat16* q_norm;
  const __nv_bfloat16* k_norm;
  float eps;
  int nq, nkv, d;
  KVView kv;
  int layer, seq, pos0;
  float* q_out;
};

struct Params {
  int M, N, K;       // N = output columns of D (SwiGLU: 2 x act columns per tile)
  int kind;
  int a_terms;       // 1 or 2
  int lo_col0;       // with 2 terms: only output tiles from this column on use A_lo
  int ksplit;        // K split into this many parts per tile (kResidual only: atomic adds)
  HeadEpi he;        // kQKVHead only
  int n_tiles_m, n_tiles_n;
  int stages;
  float* out;        // kStore: fp32 [M, ldo]; kResidual: fp32 [M, ldo] (+=)
  int ldo;
  __half* act_hi;    // kSwiGLU: fp16 [M, I] outputs (hi and lo terms)
  __half* act_lo;
  int act_ld;
  int* err;
};

// Epilogue of a QKV tile (columns [col0, col0 + BN) of the projection, whole
// heads since BN is a multiple of d) for this thread's row m. All lanes take
// part in the tensor-memory loads; only live rows store.
template <int BN>
__device__ __forceinline__ void qkv_head_epilogue(const HeadEpi& e, uint32_t taddr, int col0,
                                                  int m, bool live) {
  const int d = e.d, half = d / 2;
  const int pos = e.pos0 + m;
  for (int cb = 0; cb < BN; cb += d) {
    const int gh = (col0 + cb) / d;  // head index over q | k | v
    if (gh >= e.nq + e.nkv) {
      // v head: bf16 into the cache
      const int g = gh - e.nq - e.nkv;
      const size_t off = live ? e.kv.offset(e.layer, e.seq, pos, g) : 0;
      for (int c0 = 0; c0 < d; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(taddr + cb + c0, r);
        if (!live) continue;
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
          __align__(16) __nv_bfloat16 v[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) v[i] = __float2bfloat16_rn(__uint_as_float(r[j + i]));
          *reinterpret_cast<uint4*>(e.kv.v + off + c0 + j) = *reinterpret_cast<uint4*>(v);
        }
      }
      continue;
    }
    const bool is_q = gh < e.nq;
    const __nv_bfloat16* gain = is_q ? e.q_norm : e.k_norm;
    float ss = 0.f;
    for (int c0 = 0; c0 < d; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(taddr + cb + c0, r);
#pragma unroll
      for (int j = 0; j < 32; ++j) ss = fmaf(__uint_as_float(r[j]), __uint_as_float(r[j]), ss);
    }
    const float inv = rsqrtf(ss / (float)d + e.eps);
    const float2* cs = e.rope + (size_t)(live ? pos : 0) * half;
    float* qdst = e.q_out + (size_t)m * e.nq * d + (size_t)gh * d;
    const size_t koff = (!is_q && live) ? e.kv.offset(e.layer, e.seq, pos, gh - e.nq) : 0;
    // pairs (i, i + d/2): columns c0 .. c0+31 of the first half with the
    // same columns of the second half
    for (int c0 = 0; c0 < half; c0 += 32) {
      uint32_t lo[32], hi[32];
      tmem_ld32(taddr + cb + c0, lo);
      tmem_ld32(taddr + cb + half + c0, hi);
      if (!live) continue;
#pragma unroll
      for (int j = 0; j < 32; j += 8) {
        float olo[8], ohi[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int i = c0 + j + q;
          const float a = __uint_as_float(lo[j + q]) * inv * __bfloat162float(gain[i]);
          const float b = __uint_as_float(hi[j + q]) * inv * __bfloat162float(gain[half + i]);
          const float2 t = cs[i];
          olo[q] = a * t.x - b * t.y;
          ohi[q] = b * t.x + a * t.y;
        }
        if (is_q) {
          float* dl = qdst + c0 + j;
          float* dh = qdst + half + c0 + j;
          *reinterpret_cast<float4*>(dl) = make_float4(olo[0], olo[1], olo[2], olo[3]);
          *reinterpret_cast<float4*>(dl + 4) = make_float4(olo[4], olo[5], olo[6], olo[7]);
          *reinterpret_cast<float4*>(dh) = make_float4(ohi[0], ohi[1], ohi[2], ohi[3]);
          *reinterpret_cast<float4*>(dh + 4) = make_float4(ohi[4], ohi[5], ohi[6], ohi[7]);
        } else {
          __align__(16) __nv_bfloat16 kl[8], kh[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            kl[q] = __float2bfloat16_rn(olo[q]);
            kh[q] = __float2bfloat16_rn(ohi[q]);
          }
          *reinterpret_cast<uint4*>(e.kv.k + koff + c0 + j) = *reinterpret_cast<uint4*>(kl);
          *reinterpret_cast<uint4*>(e.kv.k + koff + half + c0 + j) = *reinterpret_cast<uint4*>(kh);
        }
      }
    }
  }
}

// BN (128 or 256): output columns per tile; the B tile is BN x 64 and the two
// fp32 accumulators take 2 x BN tensor-memory columns.
template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap map_a,
                   const __grid_constant__ CUtensorMap map_a_lo,
                   const __grid_constant__ CUtensorMap map_b,
                   const __grid_constant__ CUtensorMap map_b2) {
  pdl_trigger();
  pdl_wait();  // launched early by dependent launch: nothing before this point
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte aligned base for the swizzled tiles
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.stages;
  constexpr int kBBytes = BN * BK * 2;
  const int stage_bytes = p.a_terms * kTileBytes + kBBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * stage_bytes);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;   // [2]
  uint64_t* acc_empty = acc_full + 2;  // [2]
  uint64_t* drain = acc_empty + 2;  // MMA completion before TMEM is freed
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(drain + 1);
  uint32_t* counts = tmem_base_s + 1;  // [0] stages loaded, [1] stages consumed
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);
    }
    mbar_init(drain, 1);
    counts[0] = counts[1] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     su32(tmem_base_s)),
                 "r"(2 * BN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_base_s;

  const int n_tiles = p.n_tiles_m * p.n_tiles_n;
  const int n_units = n_tiles * p.ksplit;  // (tile, K part) work units
  const int kblocks = p.K / BK;
  const bool swiglu = p.kind == kSwiGLU;

  if (warp == 0) {
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        const int t = u / p.ksplit, kp = u % p.ksplit;
        const int mt = t % p.n_tiles_m, nt = t / p.n_tiles_m;
        const int kb0 = kblocks * kp / p.ksplit, kb1 = kblocks * (kp + 1) / p.ksplit;
        for (int kb = kb0; kb < kb1 && ok; ++kb) {
          ok = mbar_wait(&empty[s], ph ^ 1, p.err);
          if (!ok) break;
          unsigned char* st = smem + s * stage_bytes;
          const bool two = p.a_terms == 2 && nt * BN >= p.lo_col0;
          mbar_expect_tx(&full[s], stage_bytes - (p.a_terms == 2 && !two ? kTileBytes : 0));
          tma_load_2d(st, &map_a, kb * BK, mt * BM, &full[s]);
          if (two) tma_load_2d(st + kTileBytes, &map_a_lo, kb * BK, mt * BM, &full[s]);
          unsigned char* sb = st + p.a_terms * kTileBytes;
          if (swiglu) {
            // 64 gate rows then 64 up rows of the same act columns
            tma_load_2d(sb, &map_b, kb * BK, nt * (BN / 2), &full[s]);
            tma_load_2d(sb + kBBytes / 2, &map_b2, kb * BK, nt * (BN / 2), &full[s]);
          } else {
            tma_load_2d(sb, &map_b, kb * BK, nt * BN, &full[s]);
          }
          ++counts[0];
          if (++s == S) {
            s = 0;
            ph ^= 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = instr_desc(BM, BN);
      int s = 0;
      uint32_t ph = 0;
      int tcount = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++tcount) {
        const int t = u / p.ksplit, kp = u % p.ksplit;
        const int kb0 = kblocks * kp / p.ksplit, kb1 = kblocks * (kp + 1) / p.ksplit;
        const int abuf = tcount & 1;
        const uint32_t aph = (tcount >> 1) & 1;
        ok = mbar_wait(&acc_empty[abuf], aph ^ 1, p.err);
        if (!ok) break;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t d_tmem = tmem + abuf * BN;
        const bool two = p.a_terms == 2 && (t / p.n_tiles_m) * BN >= p.lo_col0;
        for (int kb = kb0; kb < kb1 && ok; ++kb) {
          ok = mbar_wait(&full[s], ph, p.err);
          if (!ok) break;
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
          unsigned char* st = smem + s * stage_bytes;
          const unsigned char* sb = st + p.a_terms * kTileBytes;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t bdesc = smem_desc(sb + k * 32);
            mma_f16(d_tmem, smem_desc(st + k * 32), bdesc, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
            if (two) mma_f16(d_tmem, smem_desc(st + kTileBytes + k * 32), bdesc, idesc, 1u);
          }
          mma_commit(&empty[s]);  // the stage is free once these MMAs have read it
          ++counts[1];
          if (++s == S) {
            s = 0;
            ph ^= 1;
          }
        }
        mma_commit(&acc_full[abuf]);  // accumulator complete
      }
      // Every MMA this thread issued has finished before TMEM is released.
      mma_commit(drain);
      const unsigned long long t0 = now_ns();
      while (!mbar_try(drain, 0))
        if (now_ns() - t0 > kTimeoutNs) break;
    }
  } else {
    // epilogue warps 2..5: TMEM lane quadrant = warp % 4
    const int quad = warp & 3;
    const int row_in_tile = quad * 32 + lane;
    int tcount = 0;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++tcount) {
      const int t = u / p.ksplit;
      const int mt = t % p.n_tiles_m, nt = t / p.n_tiles_m;
      const int abuf = tcount & 1;
      const uint32_t aph = (tcount >> 1) & 1;
      if (!mbar_wait(&acc_full[abuf], aph, p.err)) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + abuf * BN;
      const int m = mt * BM + row_in_tile;
      const bool live = m < p.M;
      if (p.kind == kQKVHead) {
        qkv_head_epilogue<BN>(p.he, taddr, nt * BN, m, live);
      } else if (!swiglu) {
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(taddr + c0, r);
          if (!live) continue;
          float* o = p.out + (size_t)m * p.ldo + nt * BN + c0;
          if (p.kind == kResidual && p.ksplit > 1) {
            // several K parts add into the same rows: vector atomics
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              atomicAdd(reinterpret_cast<float4*>(o + j),
                        make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                    __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3])));
          } else if (p.kind == kResidual) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              float4 h = *reinterpret_cast<float4*>(o + j);
              h.x += __uint_as_float(r[j]);
              h.y += __uint_as_float(r[j + 1]);
              h.z += __uint_as_float(r[j + 2]);
              h.w += __uint_as_float(r[j + 3]);
              *reinterpret_cast<float4*>(o + j) = h;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              *reinterpret_cast<float4*>(o + j) =
                  make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                              __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
          }
        }
      } else {
        // columns [0, 64) gate, [64, 128) up of act columns nt*64 + c
        for (int c0 = 0; c0 < BN / 2; c0 += 32) {
          uint32_t g[32], u[32];
          tmem_ld32(taddr + c0, g);
          tmem_ld32(taddr + BN / 2 + c0, u);
          if (!live) continue;
          const size_t off = (size_t)m * p.act_ld + nt * (BN / 2) + c0;
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            __align__(16) __half hi[8], lo[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float gv = __uint_as_float(g[j + q]), uv = __uint_as_float(u[j + q]);
              const float a = gv / (1.f + expf(-gv)) * uv;
              hi[q] = __float2half_rn(a);
              lo[q] = __float2half_rn(a - __half2float(hi[q]));
            }
            *reinterpret_cast<uint4*>(p.act_hi + off + j) = *reinterpret_cast<uint4*>(hi);
            if (p.act_lo) *reinterpret_cast<uint4*>(p.act_lo + off + j) = *reinterpret_cast<uint4*>(lo);
          }
        }
      }
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[abuf]);
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  // After a timeout: stages loaded but never consumed must land before the
  // CTA's shared memory is released (bounded wait, 10 ms each).
  if (threadIdx.x == 0 && counts[0] > counts[1]) {
    for (uint32_t k = counts[1]; k < counts[0]; ++k) {
      const unsigned long long t0 = now_ns();
      while (!mbar_try(&full[k % S], (k / S) & 1))
        if (now_ns() - t0 > 10000000ull) break;
    }
  }
  if (warp == 1) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * BN)
                 : "memory");
  }
}

}  // namespace tc

// ---------------------------------------------------------------------------
// Host side

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

}  // namespace

bool make_tmap_16(CUtensorMap* map, const void* base, long long rows, int cols, int box_rows,
                  bool bf16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
            const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {
template <int BN>
cudaError_t launch_bn(const CUtensorMap* a, const CUtensorMap* a_lo, const CUtensorMap* b,
                      const CUtensorMap* b2, int M, int N, int K, int kind, float* out, int ldo,
                      __half* act_hi, __half* act_lo, int act_ld, int* err, int num_sms,
                      cudaStream_t st, int lo_col0, const tc::HeadEpi* he) {
  static bool attr_done = false;
  if (!attr_done) {
    cudaFuncSetAttribute(tc::gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         232448);
    attr_done = true;
  }
  tc::Params p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.kind = kind;
  p.a_terms = a_lo ? 2 : 1;
  p.lo_col0 = lo_col0;
  if (he) p.he = *he;
  p.n_tiles_m = (M + tc::BM - 1) / tc::BM;
  p.n_tiles_n = N / BN;
  // Residual GEMMs with fewer tiles than SMs split K in two (atomic adds).
  p.ksplit = (kind == tc::kResidual && p.n_tiles_m * p.n_tiles_n < num_sms && (K / tc::BK) >= 8)
                 ? 2 : 1;
  const int stage_bytes = p.a_terms * tc::kTileBytes + BN * tc::BK * 2;
  p.stages = std::min(8, (232448 - 2048) / stage_bytes);
  p.out = out;
  p.ldo = ldo;
  p.act_hi = act_hi;
  p.act_lo = act_lo;
  p.act_ld = act_ld;
  p.err = err;
  const size_t smem = 1024 + (size_t)p.stages * stage_bytes + 1024;
  const int units = p.n_tiles_m * p.n_tiles_n * p.ksplit;
  const int grid = std::min(units, num_sms);
  count_launches();
  return launch_pdl(tc::gemm_tc_kernel<BN>, dim3(grid), dim3(tc::kThreads), smem, st, p, *a,
                    a_lo ? *a_lo : *a, *b, b2 ? *b2 : *b);
}
}  // namespace

// Launch one tensor-core GEMM with BN-wide output tiles (128 or 256; the B
// tensor maps must have boxes of BN rows, BN / 2 for kSwiGLU). a_lo may be
// null (one fp16 term). For kSwiGLU b2 is the up matrix and N counts
// gate+up columns (2 * I). With a_lo, output tiles from column lo_col0 on
// add the second term (0: all tiles).
cudaError_t launch_gemm_tc(const CUtensorMap* a, const CUtensorMap* a_lo, const CUtensorMap* b,
                           const CUtensorMap* b2, int M, int N, int K, int kind, float* out,
                           int ldo, __half* act_hi, __half* act_lo, int act_ld, int* err,
                           int num_sms, cudaStream_t st, int bn, int lo_col0) {
  if (bn == 256)
    return launch_bn<256>(a, a_lo, b, b2, M, N, K, kind, out, ldo, act_hi, act_lo, act_ld, err,
                          num_sms, st, lo_col0, nullptr);
  return launch_bn<128>(a, a_lo, b, b2, M, N, K, kind, out, ldo, act_hi, act_lo, act_ld, err,
                        num_sms, st, lo_col0, nullptr);
}

// The QKV GEMM of a prefill chunk with the per-head epilogue (see HeadEpi):
// rows map to positions pos0.. of sequence seq; q goes to q_out, k and v to
// the cache. bn must be a multiple of d.
cudaError_t launch_gemm_tc_qkv_heads(const CUtensorMap* a, const CUtensorMap* a_lo,
                                     const CUtensorMap* b, int M, int N, int K, int* err,
                                     int num_sms, cudaStream_t st, int bn, int lo_col0,
                                     const float2* rope, const __nv_bfloat16* q_norm,
                                     const __nv_bfloat16* k_norm, float eps, int nq, int nkv,
                                     int d, const KVView& kv, int layer, int seq, int pos0,
                                     float* q_out) {
  tc::HeadEpi he{rope, q_norm, k_norm, eps, nq, nkv, d, kv, layer, seq, pos0, q_out};
  if (bn == 256)
    return launch_bn<256>(a, a_lo, b, nullptr, M, N, K, tc::kQKVHead, nullptr, 0, nullptr,
                          nullptr, 0, err, num_sms, st, lo_col0, &he);
  return launch_bn<128>(a, a_lo, b, nullptr, M, N, K, tc::kQKVHead, nullptr, 0, nullptr, nullptr,
                        0, err, num_sms, st, lo_col0, &he);
}

}  // namespace fs
