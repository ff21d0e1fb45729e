// Causal GQA attention of a prefill chunk on the tensor cores (tcgen05 + TMEM
// + TMA), flash-attention style: the score tile S = Q K^T and the output
// accumulator O = sum P V live in tensor memory; the softmax runs in fp32
// registers with a running row maximum and row sum.
//
// One CTA per (128-query tile, query head), heaviest (latest) tiles first.
// Keys are consumed one KV page (64 positions) at a time, straight from the
// paged cache: K and V pages of one kv head are contiguous 64 x d bf16 blocks,
// loaded by TMA with 128-byte swizzle. K is the B operand of S (K-major), V
// the B operand of O (MN-major: d contiguous).
//
// Precision: Q and P enter the bf16 MMAs as two bf16 terms each (hi + lo,
// about 16 mantissa bits), so the only bf16 rounding is that of the cache
// itself; scores, softmax and O accumulate in fp32. The running maximum is
// updated lazily (only when it grows by more than 2^8 in the exp2 domain),
// which keeps every P below 256 and the final O / l exact up to rounding.
//
// Warp roles (192 threads): warp 0 TMA producer; warp 1 TMEM owner and MMA
// issuer (one lane); warps 2-5 softmax, one query row per thread (TMEM lane
// quadrant = warp % 4), then the epilogue writing O / l as fp16.
//
// Requirement: KV slots past a sequence's length hold finite values (they are
// multiplied by exact zeros); the cache is zeroed when allocated and only ever
// written with K/V rows.
#include <algorithm>

#include "runtime.h"
#include "tc_common.cuh"

namespace fs {
namespace attn_tc {

using namespace tc;

constexpr int kThreads = 192;
constexpr int kQTile = 128;
constexpr int kKTile = kPage;  // 64 keys = one KV page
constexpr float kRescaleLog2 = 8.0f;

struct Params {
  const float* q;  // [rows][nq][d] rotated queries
  __half* o;       // [rows][nq * d]
  const int32_t* block_table;
  int pages_per_seq, n_pages, nkv, nq, group;
  int layer, seq, pos0, rows, n_qt;
  int stages;
  float scale_log2;  // log2(e) / sqrt(d)
  int* err;
};

template <int D>
struct Layout {
  static constexpr int kChunks = D / 64;             // 64-element (128-byte) column chunks
  static constexpr int kQBytes = 2 * kChunks * 16384;  // Q hi, Q lo: 128 rows x 128 B per chunk
  static constexpr int kPBytes = 4 * 16384;            // P[2 buffers][hi, lo]: 128 x 64 bf16
  static constexpr int kStageBytes = 2 * kChunks * 8192;  // K and V pages: 64 rows x 128 B per chunk
  static constexpr int kTmemCols = 256;                // S[2] (64 cols each) + O (d cols)
  static constexpr int kOCol = 128;
};

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}
// hi = bf16(x), lo = bf16(x - hi) for 8 values; written as two 16-byte units.
__device__ __forceinline__ void split8(const float* x, uint4& hi, uint4& lo) {
  float h[8], l[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    h[i] = __bfloat162float(__float2bfloat16_rn(x[i]));
    l[i] = x[i] - h[i];
  }
  hi = make_uint4(pack_bf16(h[0], h[1]), pack_bf16(h[2], h[3]), pack_bf16(h[4], h[5]),
                  pack_bf16(h[6], h[7]));
  lo = make_uint4(pack_bf16(l[0], l[1]), pack_bf16(l[2], l[3]), pack_bf16(l[4], l[5]),
                  pack_bf16(l[6], l[7]));
}
// Byte offset of 16-byte unit u of row r in a 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t swz(int r, int u) {
  return (uint32_t)(r * 128 + ((u ^ (r & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attention_tc_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap map_k,
                        const __grid_constant__ CUtensorMap map_v) {
  using Lay = Layout<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = smem;
  unsigned char* sP = smem + Lay::kQBytes;
  unsigned char* sKV = sP + Lay::kPBytes;
  const int NS = p.stages;
  uint64_t* kv_full = reinterpret_cast<uint64_t*>(sKV + NS * Lay::kStageBytes);
  uint64_t* kv_empty = kv_full + NS;
  uint64_t* s_full = kv_empty + NS;  // [2]
  uint64_t* s_free = s_full + 2;     // [2]
  uint64_t* p_full = s_free + 2;     // [2]
  uint64_t* p_free = p_full + 2;     // [2]
  uint64_t* q_full = p_free + 2;
  uint64_t* o_full = q_full + 1;
  uint64_t* drain = o_full + 1;
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(drain + 1);
  uint32_t* counts = tmem_base_s + 1;  // [0] pages loaded, [1] pages waited for

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = p.n_qt - 1 - (int)blockIdx.x / p.nq;
  const int h = (int)blockIdx.x % p.nq;
  const int g = h / p.group;
  const int q0 = qt * kQTile;
  const int last_row = min(q0 + kQTile - 1, p.rows - 1);
  const int nt = (p.pos0 + last_row) / kKTile + 1;  // KV pages this tile attends

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], 128);
      mbar_init(&p_full[b], 128);
      mbar_init(&p_free[b], 1);
    }
    mbar_init(q_full, 128);
    mbar_init(o_full, 1);
    mbar_init(drain, 1);
    counts[0] = counts[1] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(tmem_base_s, Lay::kTmemCols);
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_base_s;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      for (int j = 0; j < nt; ++j) {
        const int s = j % NS;
        if (!mbar_wait(&kv_empty[s], ((j / NS) & 1) ^ 1, p.err)) break;
        int page = p.block_table[(size_t)p.seq * p.pages_per_seq + j];
        if (page < 0 || page >= p.n_pages) {
          atomicCAS(p.err, 0, kErrBounds);
          page = 0;
        }
        const int row = ((p.layer * p.n_pages + page) * p.nkv + g) * kKTile;
        unsigned char* st = sKV + s * Lay::kStageBytes;
        mbar_expect_tx(&kv_full[s], Lay::kStageBytes);
#pragma unroll
        for (int c = 0; c < Lay::kChunks; ++c) {
          tma_load_2d(st + c * 8192, &map_k, c * 64, row, &kv_full[s]);
          tma_load_2d(st + (Lay::kChunks + c) * 8192, &map_v, c * 64, row, &kv_full[s]);
        }
        ++counts[0];
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_s = instr_desc(kQTile, kKTile, true, false);
      const uint32_t id_pv = instr_desc(kQTile, D, true, true);
      const uint32_t t_o = tmem + Lay::kOCol;
      bool ok = mbar_wait(q_full, 0, p.err);
      if (ok) fence_after();
      for (int j = 0; j <= nt && ok; ++j) {
        if (j < nt) {
          const int s = j % NS, b = j & 1;
          ok = mbar_wait(&kv_full[s], (j / NS) & 1, p.err);
          if (!ok) break;
          ++counts[1];
          ok = mbar_wait(&s_free[b], ((j >> 1) & 1) ^ 1, p.err);
          if (!ok) break;
          fence_after();
          const unsigned char* kst = sKV + s * Lay::kStageBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int c = kk >> 2, off = (kk & 3) * 32;
            const uint64_t bk = smem_desc(kst + c * 8192 + off);
            mma_f16(tmem + b * kKTile, smem_desc(sQ + c * 16384 + off), bk, id_s, kk > 0 ? 1u : 0u);
            mma_f16(tmem + b * kKTile, smem_desc(sQ + (Lay::kChunks + c) * 16384 + off), bk, id_s,
                    1u);
          }
          mma_commit(&s_full[b]);
        }
        if (j >= 1) {
          const int i = j - 1, s = i % NS, b = i & 1;
          ok = mbar_wait(&p_full[b], (i >> 1) & 1, p.err);
          if (!ok) break;
          fence_after();
          const unsigned char* vst = sKV + s * Lay::kStageBytes + Lay::kChunks * 8192;
          const unsigned char* pb = sP + b * 2 * 16384;
#pragma unroll
          for (int kk = 0; kk < kKTile / 16; ++kk) {
            const uint64_t bv = smem_desc(vst + kk * 2048, 8192, 1024);
            mma_f16(t_o, smem_desc(pb + kk * 32), bv, id_pv, (i > 0 || kk > 0) ? 1u : 0u);
            mma_f16(t_o, smem_desc(pb + 16384 + kk * 32), bv, id_pv, 1u);
          }
          mma_commit(&p_free[b]);
          mma_commit(&kv_empty[s]);
        }
      }
      if (ok) mma_commit(o_full);
      // Every MMA issued has completed before TMEM is released.
      mma_commit(drain);
      const unsigned long long t0 = now_ns();
      while (!mbar_try(drain, 0))
        if (now_ns() - t0 > kTimeoutNs) break;
    }
  } else {
    // ---------------------------------------------------------------- softmax warps
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int r = q0 + row;
    const bool live = r < p.rows;
    const int qp = p.pos0 + (live ? r : p.rows - 1);  // position of this query
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;

    // Q row -> two bf16 terms in swizzled K-major layout.
    {
      const float4* src = reinterpret_cast<const float4*>(p.q + ((size_t)r * p.nq + h) * D);
#pragma unroll
      for (int c = 0; c < Lay::kChunks; ++c) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          float x[8];
          if (live) {
            const float4 a = src[c * 16 + u * 2], b4 = src[c * 16 + u * 2 + 1];
            x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
            x[4] = b4.x; x[5] = b4.y; x[6] = b4.z; x[7] = b4.w;
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] = 0.f;
          }
          uint4 hi, lo;
          split8(x, hi, lo);
          *reinterpret_cast<uint4*>(sQ + c * 16384 + swz(row, u)) = hi;
          *reinterpret_cast<uint4*>(sQ + (Lay::kChunks + c) * 16384 + swz(row, u)) = lo;
        }
      }
      fence_proxy_async();
      mbar_arrive(q_full);
    }

    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nt && ok; ++j) {
      const int b = j & 1;
      ok = mbar_wait_warp(&s_full[b], (j >> 1) & 1, p.err);
      if (!ok) break;
      fence_after();
      float x[kKTile];
      {
        uint32_t ra[32], rb[32];
        tmem_ld32(tmem + lane_off + b * kKTile, ra);
        tmem_ld32(tmem + lane_off + b * kKTile + 32, rb);
        fence_before();
        mbar_arrive(&s_free[b]);
        const int lim = qp - j * kKTile;  // keys c <= lim are visible
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          x[c] = c <= lim ? __uint_as_float(ra[c]) * p.scale_log2 : -INFINITY;
          x[c + 32] = c + 32 <= lim ? __uint_as_float(rb[c]) * p.scale_log2 : -INFINITY;
        }
      }
      float mx = x[0];
#pragma unroll
      for (int c = 1; c < kKTile; ++c) mx = fmaxf(mx, x[c]);
      const float m_new = fmaxf(m, mx);
      if (j == 0) {
        m = m_new;  // key 0 is visible to every row: finite
      } else if (__any_sync(0xffffffffu, m_new > m + kRescaleLog2)) {
        const float alpha = exp2f(m - m_new);
        // O may only be rescaled once the previous P V has landed in it.
        ok = mbar_wait_warp(&p_free[(j - 1) & 1], ((j - 1) >> 1) & 1, p.err);
        if (!ok) break;
        fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + Lay::kOCol + c0, o);
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
          tmem_st32(tmem + lane_off + Lay::kOCol + c0, o);
        }
        l *= alpha;
        m = m_new;
      }
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < kKTile; ++c) {
        x[c] = exp2f(x[c] - m);
        sum += x[c];
      }
      l += sum;
      // P buffer b is free once the P V of page j - 2 has completed.
      ok = mbar_wait_warp(&p_free[b], ((j >> 1) & 1) ^ 1, p.err);
      if (!ok) break;
      unsigned char* pb = sP + b * 2 * 16384;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        uint4 hi, lo;
        split8(x + u * 8, hi, lo);
        *reinterpret_cast<uint4*>(pb + swz(row, u)) = hi;
        *reinterpret_cast<uint4*>(pb + 16384 + swz(row, u)) = lo;
      }
      fence_proxy_async();
      fence_before();
      mbar_arrive(&p_full[b]);
    }
    if (ok) ok = mbar_wait_warp(o_full, 0, p.err);
    if (ok) {
      fence_after();
      const float inv = 1.f / l;
      __half* dst = p.o + ((size_t)r * p.nq + h) * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + Lay::kOCol + c0, o);
        if (live) {
#pragma unroll
          for (int c = 0; c < 32; c += 8) {
            __align__(16) __half v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = __float2half_rn(__uint_as_float(o[c + i]) * inv);
            *reinterpret_cast<uint4*>(dst + c0 + c) = *reinterpret_cast<uint4*>(v);
          }
        }
      }
    }
  }
  fence_before();
  __syncthreads();
  // After a timeout: pages loaded but never waited for must land before the
  // CTA's shared memory is released (bounded wait, 10 ms each).
  if (threadIdx.x == 0 && counts[0] > counts[1]) {
    for (uint32_t k = counts[1]; k < counts[0]; ++k) {
      const unsigned long long t0 = now_ns();
      while (!mbar_try(&kv_full[k % NS], (k / NS) & 1))
        if (now_ns() - t0 > 10000000ull) break;
    }
  }
  if (warp == 1) {
    fence_after();
    tmem_dealloc(tmem, Lay::kTmemCols);
  }
}

template <int D>
cudaError_t launch(const Params& p, const CUtensorMap& mk, const CUtensorMap& mv, int grid,
                   cudaStream_t st) {
  using Lay = Layout<D>;
  constexpr int kMaxSmem = 232448;
  constexpr int kFixed = 1024 + Lay::kQBytes + Lay::kPBytes + 256;
  static bool attr_done = false;
  if (!attr_done) {
    cudaFuncSetAttribute(attention_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kMaxSmem);
    attr_done = true;
  }
  Params q = p;
  q.stages = std::min(4, (kMaxSmem - kFixed) / Lay::kStageBytes);
  if (q.stages < 2) return cudaErrorInvalidValue;
  const size_t smem = kFixed + (size_t)q.stages * Lay::kStageBytes;
  count_launches();
  attention_tc_kernel<D><<<grid, kThreads, smem, st>>>(q, mk, mv);
  return cudaGetLastError();
}

}  // namespace attn_tc

bool attention_tc_supported(const Shape& s, const KVView& kv, const RowMap& map) {
  const long long kv_rows = (long long)s.L * kv.n_pages * s.nkv * kPage;
  return map.n_list == 0 && (s.d == 64 || s.d == 128) && kv_rows < (1LL << 31) &&
         s.nq % s.nkv == 0;
}

// Causal attention of `rows` consecutive positions map.pos0.. of sequence
// map.seq0 (their K/V already appended), output fp16 [rows][nq*d].
cudaError_t launch_attention_tc(const float* q, int rows, const RowMap& map, const Shape& s,
                                const KVView& kv, int layer, __half* o, int* err,
                                cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  if (!attention_tc_supported(s, kv, map)) return cudaErrorInvalidValue;
  const long long kv_rows = (long long)s.L * kv.n_pages * s.nkv * kPage;
  CUtensorMap mk, mv;
  if (!make_tmap_16(&mk, kv.k, kv_rows, s.d, kPage, true) ||
      !make_tmap_16(&mv, kv.v, kv_rows, s.d, kPage, true))
    return cudaErrorInvalidValue;
  attn_tc::Params p{};
  p.q = q;
  p.o = o;
  p.block_table = kv.block_table;
  p.pages_per_seq = kv.pages_per_seq;
  p.n_pages = kv.n_pages;
  p.nkv = s.nkv;
  p.nq = s.nq;
  p.group = s.nq / s.nkv;
  p.layer = layer;
  p.seq = map.seq0;
  p.pos0 = map.pos0;
  p.rows = rows;
  p.n_qt = (rows + attn_tc::kQTile - 1) / attn_tc::kQTile;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)s.d);
  p.err = err;
  const int grid = p.n_qt * s.nq;
  return s.d == 128 ? attn_tc::launch<128>(p, mk, mv, grid, st)
                    : attn_tc::launch<64>(p, mk, mv, grid, st);
}

}  // namespace fs
