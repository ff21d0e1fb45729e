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
// Warp roles (576 threads): warp 0 TMA producer; warp 1 TMEM owner and MMA
// issuer (one lane); warps 2-17 softmax, four warps per TMEM lane quadrant
// (= warp % 4): each thread owns one query row and a quarter of the score
// and O columns, then the epilogue writes its quarter of O / l as fp16.
//
// Requirement: KV slots past a sequence's length hold finite values (they are
// multiplied by exact zeros); the cache is zeroed when allocated and only ever
// written with K/V rows.
#include <algorithm>

#include "runtime.h"
#include "tc_common.cuh"

// Terms of the bf16 Q and P operands (2: hi + lo, 1: hi only). Two terms keep
// about 16 bits of each fp32 value; one term keeps 8 and halves the MMAs of
// the product it feeds.
#ifndef FS_ATTN_Q_TERMS
#define FS_ATTN_Q_TERMS 2
#endif
#ifndef FS_ATTN_P_TERMS
#define FS_ATTN_P_TERMS 2
#endif

namespace fs {
namespace attn_tc {

using namespace tc;

constexpr int kSoftWarps = 16;
constexpr int kGroups = kSoftWarps / 4;  // warps sharing a TMEM lane quadrant
constexpr int kSCols = 64 / kGroups;     // score columns of a page per warp
constexpr int kSoft = kSoftWarps * 32;
constexpr int kThreads = 64 + kSoft;
constexpr int kQTile = 128;
constexpr int kKTile = kPage;  // 64 keys = one KV page
constexpr float kRescaleLog2 = 8.0f;

struct Params {
  const float* q;  // [rows][nq][d] rotated queries
  __half* o;       // [rows][nq * d]
  const int32_t* block_table;
  int pages_per_seq, n_pages, nkv, nq, group;
  int layer, seq, pos0, rows, n_qt;
  float scale_log2;  // log2(e) / sqrt(d)
  int* err;
};

template <int D>
struct Layout {
  static constexpr int kChunks = D / 64;             // 64-element (128-byte) column chunks
  static constexpr int kQBytes = 2 * kChunks * 16384;  // Q hi, Q lo: 128 rows x 128 B per chunk
  static constexpr int kPBytes = 4 * 16384;            // P[2 buffers][hi, lo]: 128 x 64 bf16
  static constexpr int kPageBytes = kChunks * 8192;  // one K or V page: 64 rows x 128 B per chunk
  static constexpr int kNK = 3, kNV = 2;              // K and V ring stages
  static constexpr int kKVBytes = (kNK + kNV) * kPageBytes;
  static constexpr int kMiscBytes = 256 + 3 * kGroups * kQTile * 4;  // barriers, row max / sum
  static constexpr int kSmemBytes = 1024 + kQBytes + kPBytes + kKVBytes + kMiscBytes;
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
  pdl_trigger();
  pdl_wait();  // launched early by dependent launch: nothing before this point
  using Lay = Layout<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int NK = Lay::kNK, NV = Lay::kNV;
  unsigned char* sQ = smem;
  unsigned char* sP = smem + Lay::kQBytes;
  unsigned char* sK = sP + Lay::kPBytes;
  unsigned char* sV = sK + NK * Lay::kPageBytes;
  uint64_t* k_full = reinterpret_cast<uint64_t*>(sV + NV * Lay::kPageBytes);
  uint64_t* k_empty = k_full + NK;
  uint64_t* v_full = k_empty + NK;
  uint64_t* v_empty = v_full + NV;
  uint64_t* s_full = v_empty + NV;  // [2]
  uint64_t* s_free = s_full + 2;    // [2]
  uint64_t* p_full = s_free + 2;    // [2]
  uint64_t* p_free = p_full + 2;    // [2]
  uint64_t* q_full = p_free + 2;
  uint64_t* o_full = q_full + 1;
  uint64_t* drain = o_full + 1;
  uint32_t* tmem_base_s = reinterpret_cast<uint32_t*>(drain + 1);
  uint32_t* counts = tmem_base_s + 1;  // K pages loaded / waited, V pages loaded / waited
  float(*red_max)[kGroups][kQTile] = reinterpret_cast<float(*)[kGroups][kQTile]>(
      reinterpret_cast<unsigned char*>(k_full) + 256);  // [page parity][group][row]
  float(*red_sum)[kQTile] = reinterpret_cast<float(*)[kQTile]>(red_max + 2);  // [group][row]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = p.n_qt - 1 - (int)blockIdx.x / p.nq;
  const int h = (int)blockIdx.x % p.nq;
  const int g = h / p.group;
  const int q0 = qt * kQTile;
  const int last_row = min(q0 + kQTile - 1, p.rows - 1);
  const int nt = (p.pos0 + last_row) / kKTile + 1;  // KV pages this tile attends

  if (threadIdx.x == 0) {
    for (int s = 0; s < NK; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], kSoft);
      mbar_init(&p_full[b], kSoft);
      mbar_init(&p_free[b], 1);
    }
    mbar_init(q_full, kSoft);
    mbar_init(o_full, 1);
    mbar_init(drain, 1);
    counts[0] = counts[1] = counts[2] = counts[3] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(tmem_base_s, Lay::kTmemCols);
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_base_s;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    // Lane 0 streams the K pages, lane 1 the V pages, each at the pace of its
    // own ring: the next K page never waits for a V slot.
    if (lane < 2) {
      const bool is_k = lane == 0;
      const int NS = is_k ? NK : NV;
      uint64_t* fullb = is_k ? k_full : v_full;
      uint64_t* emptyb = is_k ? k_empty : v_empty;
      unsigned char* ring = is_k ? sK : sV;
      const CUtensorMap* map = is_k ? &map_k : &map_v;
      for (int j = 0; j < nt; ++j) {
        int page = p.block_table[(size_t)p.seq * p.pages_per_seq + j];
        if (page < 0 || page >= p.n_pages) {
          atomicCAS(p.err, 0, kErrBounds);
          page = 0;
        }
        const int row = ((p.layer * p.n_pages + page) * p.nkv + g) * kKTile;
        const int st = j % NS;
        if (!mbar_wait(&emptyb[st], ((j / NS) & 1) ^ 1, p.err)) break;
        mbar_expect_tx(&fullb[st], Lay::kPageBytes);
#pragma unroll
        for (int c = 0; c < Lay::kChunks; ++c)
          tma_load_2d(ring + st * Lay::kPageBytes + c * 8192, map, c * 64, row, &fullb[st]);
        ++counts[is_k ? 0 : 2];
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
          const int sk = j % NK, b = j & 1;
          ok = mbar_wait(&k_full[sk], (j / NK) & 1, p.err);
          if (!ok) break;
          ++counts[1];
          ok = mbar_wait(&s_free[b], ((j >> 1) & 1) ^ 1, p.err);
          if (!ok) break;
          fence_after();
          const unsigned char* kst = sK + sk * Lay::kPageBytes;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int c = kk >> 2, off = (kk & 3) * 32;
            const uint64_t bk = smem_desc(kst + c * 8192 + off);
            mma_f16(tmem + b * kKTile, smem_desc(sQ + c * 16384 + off), bk, id_s, kk > 0 ? 1u : 0u);
            if (FS_ATTN_Q_TERMS == 2)
              mma_f16(tmem + b * kKTile, smem_desc(sQ + (Lay::kChunks + c) * 16384 + off), bk,
                      id_s, 1u);
          }
          mma_commit(&s_full[b]);
          mma_commit(&k_empty[sk]);
        }
        if (j >= 1) {
          const int i = j - 1, sv = i % NV, b = i & 1;
          ok = mbar_wait(&v_full[sv], (i / NV) & 1, p.err);
          if (!ok) break;
          ++counts[3];
          ok = mbar_wait(&p_full[b], (i >> 1) & 1, p.err);
          if (!ok) break;
          fence_after();
          const unsigned char* vst = sV + sv * Lay::kPageBytes;
          const unsigned char* pb = sP + b * 2 * 16384;
#pragma unroll
          for (int kk = 0; kk < kKTile / 16; ++kk) {
            const uint64_t bv = smem_desc(vst + kk * 2048, 8192, 1024);
            mma_f16(t_o, smem_desc(pb + kk * 32), bv, id_pv, (i > 0 || kk > 0) ? 1u : 0u);
            if (FS_ATTN_P_TERMS == 2) mma_f16(t_o, smem_desc(pb + 16384 + kk * 32), bv, id_pv, 1u);
          }
          mma_commit(&p_free[b]);
          mma_commit(&v_empty[sv]);
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
    // kGroups warps per TMEM lane quadrant: warp group g owns score columns
    // [g * kSCols, (g + 1) * kSCols) of each page and the same share of the O
    // columns. The row maximum is combined through shared memory (one reducing
    // barrier of the quadrant's warps per page).
    const int quad = warp & 3;
    const int grp = (warp - 2) >> 2;
    const int row = quad * 32 + lane;
    const int r = q0 + row;
    const bool live = r < p.rows;
    const int qp = p.pos0 + (live ? r : p.rows - 1);  // position of this query
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    constexpr int kOCols = D / kGroups;           // O columns per warp
    constexpr int kOC = kOCols < 32 ? kOCols : 32;  // TMEM columns per load
    auto pair_sync = [&]() {
      asm volatile("bar.sync %0, %1;" ::"r"(1 + quad), "n"(32 * kGroups) : "memory");
    };
    auto pair_or = [&](int id, bool v) -> bool {
      uint32_t r;
      asm volatile(
          "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, %3, p;\n"
          " selp.u32 %0, 1, 0, q;\n}\n"
          : "=r"(r)
          : "r"((uint32_t)v), "r"(id), "n"(32 * kGroups)
          : "memory");
      return r != 0;
    };

    // Q row -> two bf16 terms in swizzled K-major layout (this warp's share of the units).
    {
      const float4* src = reinterpret_cast<const float4*>(p.q + ((size_t)r * p.nq + h) * D);
      constexpr int kUnits = Lay::kChunks * 8;  // 16-byte units of a row
#pragma unroll
      for (int uu = 0; uu < kUnits / kGroups; ++uu) {
        const int un = grp * (kUnits / kGroups) + uu;
        const int c = un >> 3, u = un & 7;
        float x[8];
        if (live) {
          // the softmax scale (log2 e / sqrt d) is folded into Q
          const float4 a = src[un * 2], b4 = src[un * 2 + 1];
          const float sc = p.scale_log2;
          x[0] = a.x * sc; x[1] = a.y * sc; x[2] = a.z * sc; x[3] = a.w * sc;
          x[4] = b4.x * sc; x[5] = b4.y * sc; x[6] = b4.z * sc; x[7] = b4.w * sc;
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) x[i] = 0.f;
        }
        uint4 hi, lo;
        split8(x, hi, lo);
        *reinterpret_cast<uint4*>(sQ + c * 16384 + swz(row, u)) = hi;
        *reinterpret_cast<uint4*>(sQ + (Lay::kChunks + c) * 16384 + swz(row, u)) = lo;
      }
      fence_proxy_async();
      mbar_arrive(q_full);
    }

    float m = -INFINITY, l = 0.f;  // l: this warp's columns only
    bool ok = true;
    // The two warps of a quadrant pair leave the loop together: every pass
    // ends in one reducing barrier that ORs their failure flags (a timed-out
    // warp skips the work but still takes part).
    for (int j = 0; j < nt; ++j) {
      const int b = j & 1;
      float x[kSCols];
      float mx = -INFINITY;
      if (ok) ok = mbar_wait_warp(&s_full[b], (j >> 1) & 1, p.err);
      if (ok) {
        fence_after();
        uint32_t ra[kSCols];
        tmem_ld(tmem + lane_off + b * kKTile + grp * kSCols, ra);
        fence_before();
        mbar_arrive(&s_free[b]);
        const int lim = qp - j * kKTile - grp * kSCols;  // columns c <= lim are visible
        if (__all_sync(0xffffffffu, lim >= kSCols - 1)) {  // below the diagonal: nothing masked
#pragma unroll
          for (int c = 0; c < kSCols; ++c) x[c] = __uint_as_float(ra[c]);
        } else {
#pragma unroll
          for (int c = 0; c < kSCols; ++c) x[c] = c <= lim ? __uint_as_float(ra[c]) : -INFINITY;
        }
        float mx4[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
        for (int c = 4; c < kSCols; c += 4)
#pragma unroll
          for (int i = 0; i < 4; ++i) mx4[i] = fmaxf(mx4[i], x[c + i]);
        mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      }
      red_max[b][grp][row] = mx;
      if (pair_or(1 + quad, !ok)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int g2 = 0; g2 < kGroups; ++g2) mx = fmaxf(mx, red_max[b][g2][row]);
      const float m_new = fmaxf(m, mx);
      if (j == 0) {
        m = m_new;  // key 0 is visible to every row: finite
      } else if (__any_sync(0xffffffffu, m_new > m + kRescaleLog2)) {
        // The quadrant's warps see the same rows and maxima: same decision.
        const float alpha = exp2f(m - m_new);
        // O may only be rescaled once the previous P V has landed in it.
        if (!mbar_wait_warp(&p_free[(j - 1) & 1], ((j - 1) >> 1) & 1, p.err)) {
          ok = false;
          continue;
        }
        fence_after();
#pragma unroll 1
        for (int c0 = grp * kOCols; c0 < (grp + 1) * kOCols; c0 += kOC) {
          uint32_t o[kOC];
          tmem_ld(tmem + lane_off + Lay::kOCol + c0, o);
#pragma unroll
          for (int c = 0; c < kOC; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
          tmem_st(tmem + lane_off + Lay::kOCol + c0, o);
        }
        l *= alpha;
        m = m_new;
      }
      float sm4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < kSCols; c += 4)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          x[c + i] = exp2f(x[c + i] - m);
          sm4[i] += x[c + i];
        }
      l += (sm4[0] + sm4[1]) + (sm4[2] + sm4[3]);
      // P buffer b is free once the P V of page j - 2 has completed.
      if (!mbar_wait_warp(&p_free[b], ((j >> 1) & 1) ^ 1, p.err)) {
        ok = false;
        continue;
      }
      unsigned char* pb = sP + b * 2 * 16384;
#pragma unroll
      for (int u = 0; u < kSCols / 8; ++u) {
        uint4 hi, lo;
        split8(x + u * 8, hi, lo);
        *reinterpret_cast<uint4*>(pb + swz(row, grp * (kSCols / 8) + u)) = hi;
        *reinterpret_cast<uint4*>(pb + 16384 + swz(row, grp * (kSCols / 8) + u)) = lo;
      }
      fence_proxy_async();
      fence_before();
      mbar_arrive(&p_full[b]);
    }
    // Full row sum from the two halves (uniform control flow for the barrier:
    // a timed-out warp still takes part).
    red_sum[grp][row] = l;
    pair_sync();
    float l_row = 0.f;
#pragma unroll
    for (int g2 = 0; g2 < kGroups; ++g2) l_row += red_sum[g2][row];
    if (ok) ok = mbar_wait_warp(o_full, 0, p.err);
    if (ok) {
      fence_after();
      const float inv = 1.f / l_row;
      __half* dst = p.o + ((size_t)r * p.nq + h) * D;
#pragma unroll 1
      for (int c0 = grp * kOCols; c0 < (grp + 1) * kOCols; c0 += kOC) {
        uint32_t o[kOC];
        tmem_ld(tmem + lane_off + Lay::kOCol + c0, o);
        if (live) {
#pragma unroll
          for (int c = 0; c < kOC; c += 8) {
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
  if (threadIdx.x == 0) {
    for (uint32_t k = counts[1]; k < counts[0]; ++k) {
      const unsigned long long t0 = now_ns();
      while (!mbar_try(&k_full[k % NK], (k / NK) & 1))
        if (now_ns() - t0 > 10000000ull) break;
    }
    for (uint32_t k = counts[3]; k < counts[2]; ++k) {
      const unsigned long long t0 = now_ns();
      while (!mbar_try(&v_full[k % NV], (k / NV) & 1))
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
  static_assert(Lay::kSmemBytes <= 232448, "shared memory budget");
  static bool attr_done = false;
  if (!attr_done) {
    cudaFuncSetAttribute(attention_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         Lay::kSmemBytes);
    attr_done = true;
  }
  const size_t smem = Lay::kSmemBytes;
  const Params& q = p;
  count_launches();
  return launch_pdl(attention_tc_kernel<D>, dim3(grid), dim3(kThreads), smem, st, q, mk, mv);
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
