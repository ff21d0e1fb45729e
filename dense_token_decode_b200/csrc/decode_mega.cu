// Persistent decode forward: one cooperative launch runs every block and the
// LM head of one decode step for a batch of up to 4 sequences.
//
// Layout of the work. Each CTA (one per SM) owns a contiguous slice of the
// rows of every weight matrix. A producer warp streams the CTA's slices —
// QKV rows, the old K/V pages of the CTA's attention items, O rows, gate/up
// row pairs, down rows, per layer, then its rows of the tied embedding for
// the LM head — through a ring of shared-memory stages, weights with
// cp.async.bulk and K/V with TMA tensor copies (128-byte swizzle, for the
// tensor cores). Weights do not depend on activations, so the producer runs
// ahead across phase and layer boundaries and HBM never waits for the
// dependency chain.
//
// Eleven consumer warps compute: chunk i of the stream (weights or K/V)
// belongs to warp i mod 11, which alone computes it and releases its stage.
// Activations move between CTAs as 64-bit
// words (fp32 value | 32-bit tag): a consumer polls the words it needs until
// their tag is the one of the current phase, so there is no grid barrier and
// no separate flag. Tags grow monotonically across steps; nothing is reset.
//
// Phases of block l (tag t_l,p): P1 RMSNorm + QKV rows -> xq; P2 attention
// items (b, kv head g, split s): q/k head RMSNorm + RoPE, append of the new
// K/V to the page, online-softmax attention over the split's keys on the
// tensor cores (one owner warp per 32-key chunk, mma.sync), merge of the
// warps' states, merge of splits by the last arriving item -> xo;
// P3 O rows + residual -> xh0;
// P4 RMSNorm + gate/up pairs + SwiGLU -> xa; P5 down rows + residual -> xh1.
// LM head: final RMSNorm, logits of the CTA's vocab rows, greedy key (value,
// lowest id) folded with a 64-bit atomicMax; the last CTA writes the ids.
//
// Every wait is bounded by %globaltimer; on timeout the CTA records
// kErrTimeout in the error word, stops waiting, drains its own bulk copies
// and returns.
#include <algorithm>

#include "runtime.h"
#include "tc_common.cuh"

namespace fs {
namespace mega {

constexpr int kConsumerWarps = 11;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;  // + producer warp
constexpr int kMaxB = 4;
constexpr int kWeightBytes = 16384;             // weight bytes of one stage
constexpr int kStageBytes = kWeightBytes + 1024; // + Q8_0 scales
constexpr int kMaxStages = 16;

enum Phase { kQKV = 0, kAttn, kO, kGU, kDown, kLM };

struct Params {
  int L, H, nq, nkv, d, I, V;
  float eps;
  int q8;
  const LayerDev* layers;
  const __nv_bfloat16* embed;
  const __nv_bfloat16* final_norm;
  const float2* rope;
  KVView kv;
  int B;
  int seq[kMaxB];
  int pos[kMaxB];
  const int32_t* tokens;
  unsigned long long* xq;   // [B][(nq+2nkv)d]
  unsigned long long* xo;   // [B][nq d]
  unsigned long long* xh0;  // [B][H]
  unsigned long long* xh1;  // [B][H]
  unsigned long long* xa;   // [B][I]
  float* part;              // [B][nkv][splits][rep][d+2]
  unsigned int* split_cnt;  // [B][nkv]
  unsigned long long* am_key;  // [B]
  unsigned int* am_cnt;
  uint32_t tag0;
  int n_splits;
  int l0, l1;
  const float* h_in;  // optional input rows [B][H] (instead of the embedding)
  float* h_out;       // optional output rows [B][H] after block l1-1
  int run_head;
  float* logits;
  int32_t* argmax;
  float* capture;
  int capture_stride;
  int* err;
  int* abort_flag;  // set on a timeout: every wait gives up
  unsigned long long wait_ns;  // limit of every wait
  int withhold_layer;          // debug: the Q/K/V rows of this block are never published
  unsigned long long* trace;  // optional: clock64 stamps [G][L+1][16]; tail row 12..15 time base
  int n_stages;
  // smem carve-up (bytes)
  int off_hs, off_xs, off_attn, off_bar, off_misc, off_tab;
  int bt_in_smem;  // block-table rows of the batch copied to shared memory
};

// Shared-memory copies of the per-layer weight pointers and of the batch's
// block-table rows: the producer thread looks them up for every chunk, and a
// global-memory round trip there would stall the whole weight stream.
__device__ __forceinline__ const LayerDev* layers_s(const Params& p) {
  extern __shared__ __align__(1024) unsigned char smem_base[];
  return reinterpret_cast<const LayerDev*>(smem_base + p.off_tab);
}
__device__ __forceinline__ size_t kv_off(const Params& p, int layer, int b, int pos, int g) {
  extern __shared__ __align__(1024) unsigned char smem_base[];
  int page;
  if (p.bt_in_smem) {
    const int32_t* bt = reinterpret_cast<const int32_t*>(
        smem_base + p.off_tab + (size_t)p.L * sizeof(LayerDev));
    page = bt[b * p.kv.pages_per_seq + pos / kPage];
  } else {
    page = p.kv.block_table[(size_t)p.seq[b] * p.kv.pages_per_seq + pos / kPage];
  }
  return (size_t)layer * p.kv.layer_elems() +
         (((size_t)page * p.kv.n_kv_heads + g) * kPage + (pos % kPage)) * p.kv.head_dim;
}

// ---------------------------------------------------------------------------
// PTX helpers

__device__ __forceinline__ uint32_t su32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(su32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(su32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(su32(dst)),
      "l"(src), "r"(bytes), "r"(su32(bar)), "l"(policy)
      : "memory");
}
__device__ __forceinline__ unsigned long long ld_tag(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_tag(unsigned long long* p, float v, uint32_t tag) {
  const unsigned long long w = ((unsigned long long)tag << 32) | __float_as_uint(v);
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
__device__ __forceinline__ unsigned long long now_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory");
}
// Barrier of the consumer warps that also ORs a flag over them, so that a
// decision to stop (a timeout seen by some threads) is taken by all at once.
__device__ __forceinline__ bool consumer_sync_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 1, %2, p;\n"
      " selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kConsumers)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ bool aborted(const int* flag) {
  return *reinterpret_cast<const volatile int*>(flag) != 0;
}
__device__ __forceinline__ void raise_timeout(const Params& p) {
  atomicExch(p.abort_flag, 1);
  atomicCAS(p.err, 0, kErrTimeout);
}
__device__ __forceinline__ float lo16(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float hi16(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// Tensor-core helpers of the attention items: ldmatrix (x4, plain and
// transposed), mma.sync m16n8k16 bf16 -> fp32, and bf16 pairs.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// bf16 bits of x (round to nearest even), and of the remainder x - bf16(x)
__device__ __forceinline__ uint32_t bf16_bits(float x) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(x));
}
__device__ __forceinline__ uint32_t bf16_term(float x, bool lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(x);
  return lo ? bf16_bits(x - __bfloat162float(h)) : (uint32_t)__bfloat16_as_ushort(h);
}

// ---------------------------------------------------------------------------
// Shapes of the chunk stream (identical in producer and consumers)

struct ChunkShape {
  int rows;  // weight rows per chunk (gate/up: pairs), at most one per consumer warp
};

// The largest power of two of whole rows (gate/up: row pairs) that fits one
// stage, at most 8 rows or 4 pairs (one warp finishes at most 8 dot products
// per chunk).
__host__ __device__ inline ChunkShape chunk_shape(int K, bool q8, bool pair) {
  const int row_bytes = (q8 ? K : 2 * K) * (pair ? 2 : 1);
  const int cap = pair ? 4 : 8;
  int rows = 1;
  while (rows * 2 <= cap && rows * 2 * row_bytes <= kWeightBytes) rows *= 2;
  return ChunkShape{rows * row_bytes <= kWeightBytes ? rows : 0};
}

__host__ __device__ inline int keys_per_chunk(int d) { return kWeightBytes / (4 * d); }

__host__ __device__ inline void slice(int N, int G, int c, int& a, int& b) {
  a = (int)((long long)N * c / G);
  b = (int)((long long)N * (c + 1) / G);
}

// Attention items of CTA c: [ia, ib).
__host__ __device__ inline void items_of(int n_items, int G, int c, int& ia, int& ib) {
  ia = (int)(((long long)c * n_items + G - 1) / G);
  ib = (int)(((long long)(c + 1) * n_items + G - 1) / G);
  if (ib > n_items) ib = n_items;
}

struct Item {
  int b, g, s, j0, j1;  // keys [j0, j1) of row b's context
  bool owner;           // holds the new position
};

__device__ inline Item item_desc(const Params& p, int it) {
  Item x;
  const int ns = p.n_splits;
  x.b = it / (p.nkv * ns);
  x.g = (it / ns) % p.nkv;
  x.s = it % ns;
  const int C = p.pos[x.b] + 1;
  const int kps = (C + ns - 1) / ns;
  x.j0 = min(C, x.s * kps);
  x.j1 = min(C, x.j0 + kps);
  x.owner = x.j0 <= p.pos[x.b] && p.pos[x.b] < x.j1;
  return x;
}

// Source of weight row n of a phase (QKV rows span wq|wk|wv).
__device__ inline const void* row_src(const Params& p, int phase, int layer, int n, int K,
                                      const __half** scale_row, int* limit) {
  const LayerDev& Lw = layers_s(p)[layer];
  int which = 0, local = n, end = 0;
  const int qd = p.nq * p.d, kvd = p.nkv * p.d;
  switch (phase) {
    case kQKV:
      if (n < qd) {
        which = kWq;
        end = qd;
      } else if (n < qd + kvd) {
        which = kWk;
        local = n - qd;
        end = qd + kvd;
      } else {
        which = kWv;
        local = n - qd - kvd;
        end = qd + 2 * kvd;
      }
      break;
    case kO: which = kWo; end = p.H; break;
    case kGU: which = kWg; end = p.I; break;
    case kDown: which = kWd; end = p.H; break;
    default: break;
  }
  *limit = end;
  if (phase == kLM) {
    *scale_row = nullptr;
    *limit = p.V;
    return p.embed + (size_t)n * K;
  }
  if (p.q8) {
    *scale_row = Lw.s[which] + (size_t)local * (K / 32);
    return static_cast<const int8_t*>(Lw.w[which]) + (size_t)local * K;
  }
  *scale_row = nullptr;
  return static_cast<const __nv_bfloat16*>(Lw.w[which]) + (size_t)local * K;
}

// End of the weight chunk that starts at row n of a phase slice ending at b:
// at most cs.rows rows, never across the wq|wk|wv boundaries.
__device__ inline int chunk_end(const Params& p, int phase, int n, int b, ChunkShape cs) {
  int e = min(b, n + cs.rows);
  if (phase == kQKV) {
    const int qd = p.nq * p.d, kvd = p.nkv * p.d;
    if (n < qd) e = min(e, qd);
    else if (n < qd + kvd) e = min(e, qd + kvd);
  }
  return e;
}

// The chunk walk: calls v.gemv(phase, layer, n0, nr, K, cs) for each weight
// chunk, v.attn_begin/kv/attn_end for attention items and v.phase_begin at
// the start of each phase with work.
template <class Vis>
__device__ void walk(const Params& p, int c, int G, Vis& v) {
  const int qkvd = (p.nq + 2 * p.nkv) * p.d;
  const int n_items = p.B * p.nkv * p.n_splits;
  const int kpc = keys_per_chunk(p.d);
  for (int l = p.l0; l < p.l1 && !v.stop(); ++l) {
    // P1: QKV rows
    {
      int a, b;
      slice(qkvd, G, c, a, b);
      const ChunkShape cs = chunk_shape(p.H, p.q8, false);
      if (a < b) {
        v.phase_begin(kQKV, l);
        v.gemv_phase(kQKV, l, a, b, p.H, cs);
      }
    }
    // P2: attention items
    {
      int ia, ib;
      items_of(n_items, G, c, ia, ib);
      for (int it = ia; it < ib; ++it) {
        const Item x = item_desc(p, it);
        v.attn_begin(l, it, x);
        const int old_end = min(x.j1, p.pos[x.b]);
        for (int j = x.j0; j < old_end;) {
          const int e = min(old_end, (j / kpc + 1) * kpc);
          v.kv(l, x, j, e - j);
          j = e;
        }
        v.attn_end(l, it, x);
      }
    }
    // P3: O rows, P4: gate/up pairs, P5: down rows
    const int phases[3] = {kO, kGU, kDown};
    for (int q = 0; q < 3; ++q) {
      const int ph = phases[q];
      const int N = (ph == kGU) ? p.I : p.H;
      const int K = (ph == kO) ? p.nq * p.d : (ph == kDown ? p.I : p.H);
      const ChunkShape cs = chunk_shape(K, p.q8, ph == kGU);
      int a, b;
      slice(N, G, c, a, b);
      if (a < b) {
        v.phase_begin(ph, l);
        v.gemv_phase(ph, l, a, b, K, cs);
      }
    }
    v.end_layer();
  }
  if (p.run_head && !v.stop()) {
    int a, b;
    slice(p.V, G, c, a, b);
    const ChunkShape cs = chunk_shape(p.H, false, false);
    if (a < b) {
      v.phase_begin(kLM, p.l1 - 1);
      v.gemv_phase(kLM, p.l1 - 1, a, b, p.H, cs);
    }
  }
}

struct Ring {
  unsigned char* stages;
  uint64_t* full;
  uint64_t* empty;
  int n;
};

// ---------------------------------------------------------------------------
// Producer: issues the bulk copies of every chunk, in walk order.

struct Producer {
  const Params& p;
  Ring r;
  uint64_t policy;
  unsigned int i = 0;  // chunks issued
  int stage = 0;       // i % ring size
  uint32_t parity = 1; // waits for the opposite phase first: fresh slots are free
  bool quit = false;
  bool lm_started = false;

  const CUtensorMap* tm_k;  // the KV cache as [rows][d] bf16, 32 x 64 boxes, 128-byte swizzle
  const CUtensorMap* tm_v;
  __device__ Producer(const Params& pp, Ring rr, const CUtensorMap* mk, const CUtensorMap* mv)
      : p(pp), r(rr), tm_k(mk), tm_v(mv) {
    policy = evict_first_policy();
  }
  __device__ bool stop() const { return quit; }
  __device__ __forceinline__ void advance() {
    ++i;
    if (++stage == r.n) {
      stage = 0;
      parity ^= 1u;
    }
  }

  __device__ unsigned char* acquire(uint32_t bytes) {
    const int s = stage;
    unsigned long long t0 = 0;
    int spins = 0;
    while (!mbar_test(&r.empty[s], parity)) {
      // The clock only starts after many failed polls: reading it is not free.
      if ((++spins & 15) == 0) {
        if (t0 == 0) t0 = now_ns();
        if (aborted(p.abort_flag) || now_ns() - t0 > p.wait_ns) {
          if (!aborted(p.abort_flag)) raise_timeout(p);
          quit = true;
          return nullptr;
        }
      }
    }
    mbar_expect_tx(&r.full[s], bytes);
    return r.stages + (size_t)s * kStageBytes;
  }

  __device__ __forceinline__ void gemv_phase(int ph, int layer, int a, int b, int K, ChunkShape cs) {
    for (int n = a; n < b && !quit;) {
      const int e = chunk_end(p, ph, n, b, cs);
      gemv(ph, layer, n, e - n, K, cs);
      n = e;
    }
  }
  __device__ void phase_begin(int, int) {}
  __device__ void end_layer() {}
  __device__ void attn_begin(int, int, const Item&) {}
  __device__ void attn_end(int, int, const Item&) {}

  __device__ void gemv(int phase, int layer, int n0, int nr, int K, ChunkShape cs) {
    if (quit) return;
    if (p.trace && phase == kLM) {
      unsigned long long* t = p.trace + ((size_t)blockIdx.x * (p.L + 1) + p.L) * 16;
      if (!lm_started) t[2] = clock64();
      lm_started = true;
    }
    const bool pair = phase == kGU;
    const bool q8 = p.q8 && phase != kLM;
    const uint32_t rb = q8 ? K : 2 * K;
    const uint32_t sb = q8 ? K / 16 : 0;  // scale bytes per row
    const uint32_t bytes = (pair ? 2 : 1) * nr * (rb + sb);
    unsigned char* st = acquire(bytes);
    if (!st) return;
    const __half* sr;
    int lim;
    const void* src = row_src(p, phase, layer, n0, K, &sr, &lim);
    uint64_t* bar = &r.full[stage];
    bulk_load(st, src, nr * rb, bar, policy);
    if (q8) bulk_load(st + kWeightBytes, sr, nr * sb, bar, policy);
    if (pair) {
      const LayerDev& Lw = layers_s(p)[layer];
      if (q8) {
        bulk_load(st + cs.rows * rb, static_cast<const int8_t*>(Lw.w[kWu]) + (size_t)n0 * K,
                  nr * rb, bar, policy);
        bulk_load(st + kWeightBytes + cs.rows * sb, Lw.s[kWu] + (size_t)n0 * (K / 32), nr * sb,
                  bar, policy);
      } else {
        bulk_load(st + cs.rows * rb,
                  static_cast<const __nv_bfloat16*>(Lw.w[kWu]) + (size_t)n0 * K, nr * rb, bar,
                  policy);
      }
    }
    advance();
  }

  // A KV chunk: keys [j, j + nk) of the item as K and V tiles in the 128-byte
  // swizzled layout the tensor-core attention reads. TMA boxes of 32 rows x
  // 64 dims: one per 32 keys and 64 dims of the chunk's kpc-key tile (rows
  // past nk are loaded too: finite cache contents, masked by the consumer;
  // rows past the cache read as zero).
  __device__ void kv(int layer, const Item& x, int j, int nk) {
    if (quit) return;
    unsigned char* st = acquire(kWeightBytes);
    if (!st) return;
    const int row = (int)(kv_off(p, layer, x.b, j, x.g) / (size_t)p.d);
    const int kpc = keys_per_chunk(p.d);
    uint64_t* bar = &r.full[stage];
    for (int cb = 0; cb < p.d / 64; ++cb)
      for (int rb = 0; rb < kpc / 32; ++rb) {
        const int off = cb * kpc * 128 + rb * 32 * 128;
        tc::tma_load_2d(st + off, tm_k, cb * 64, row + rb * 32, bar);
        tc::tma_load_2d(st + kWeightBytes / 2 + off, tm_v, cb * 64, row + rb * 32, bar);
      }
    (void)nk;
    advance();
  }
};

// ---------------------------------------------------------------------------
// Consumers

template <int NB, bool Q8W>
struct Consumer {
  const Params& p;
  Ring r;
  unsigned char* smem;
  float* hs;  // [B][H] block input / mid residual
  float* xs;  // [B][max K] GEMV operand
  float* at;    // attention scratch
  unsigned long long wbest[kMaxB] = {0ull, 0ull, 0ull, 0ull};  // this lane's greedy keys
  unsigned long long* best;  // [kMaxB] greedy keys of this CTA
  int* flag;
  unsigned int i = 0;  // chunks consumed
  int stage = 0;       // i % ring size
  uint32_t parity = 0; // (i / ring size) & 1
  bool quit = false;
  int tid, warp, lane;
  int G, cta;
  // attention state (per warp, registers)
  // attention state of the lane's head (lane % 4 < rep) on the tensor cores
  uint32_t qb[8][2];  // B fragments of q (hi, lo terms per head) per 16-dim step
  float mh, lh;       // running maximum and sum of the lane's head
  float o[8][4];      // C fragments of O^T per 16-dim tile

  __device__ Consumer(const Params& pp, Ring rr, unsigned char* sm) : p(pp), r(rr), smem(sm) {
    hs = reinterpret_cast<float*>(sm + p.off_hs);
    xs = reinterpret_cast<float*>(sm + p.off_xs);
    at = reinterpret_cast<float*>(sm + p.off_attn);
    best = reinterpret_cast<unsigned long long*>(sm + p.off_misc);
    flag = reinterpret_cast<int*>(sm + p.off_misc + 8 * kMaxB);
    tid = threadIdx.x;
    warp = tid >> 5;
    lane = tid & 31;
    G = gridDim.x;
    cta = blockIdx.x;
    cur_layer = p.l0;
  }
  __device__ bool stop() const { return quit; }

  // Timestamp slot k of (this CTA, layer) into the optional trace.
  __device__ void tr(int layer, int k) {
    if (p.trace && tid == 0) p.trace[((size_t)cta * (p.L + 1) + layer) * 16 + k] = clock64();
  }

  __device__ uint32_t tag(int layer, int ph) const {
    return p.tag0 + 5u * (uint32_t)(layer - p.l0) + (uint32_t)ph;
  }

  // Wait for the ring stage of the next chunk. On a timeout the thread sets
  // quit and carries on with whatever the stage holds until the next
  // reducing barrier makes the decision CTA-wide.
  //
  // A parity wait only tells two consecutive phases apart. A warp skips the
  // chunks it does not own, so it can reach chunk i while chunk i - n (same
  // stage, n = ring size) is still in flight; with n below the number of
  // consumer warps nothing orders the two. The stage's full barrier is then
  // in chunk i - n's phase, whose parity is the opposite of chunk i's, and a
  // parity test for chunk i reads that pending phase as the completed one
  // before it: the warp would compute on stale bytes and release the stage a
  // second time. So the warp first waits until chunk i - n has been released
  // (its empty phase, which only completes after chunk i - n's full phase
  // did and cannot advance further before this warp releases chunk i); after
  // that the full barrier can only be in chunk i's phase.
  __device__ const unsigned char* stage_wait() {
    const int s = stage;
    unsigned long long t0 = 0;
    int spins = 0;
    // Every lane observes the barrier itself (that is what makes the bulk
    // copy's bytes visible to it); the give-up decision is lane 0's, so the
    // warp stays converged for the shuffles that follow.
    while (true) {
      const bool ok =
          quit || (mbar_test(&r.empty[s], parity ^ 1u) && mbar_test(&r.full[s], parity));
      if (__all_sync(0xffffffffu, ok)) break;
      if ((++spins & 15) == 0) {
        int bad = 0;
        if (lane == 0) {
          if (t0 == 0) t0 = now_ns();
          bad = aborted(p.abort_flag) || now_ns() - t0 > p.wait_ns;
        }
        bad = __shfl_sync(0xffffffffu, bad, 0);
        if (bad) {
          if (lane == 0 && !aborted(p.abort_flag)) raise_timeout(p);
          quit = true;
        }
      }
    }
    return r.stages + (size_t)s * kStageBytes;
  }
  __device__ void stage_release() {
    __syncwarp();
    if (lane == 0) mbar_arrive(&r.empty[stage]);
  }
  __device__ __forceinline__ void advance() {
    ++i;
    if (++stage == r.n) {
      stage = 0;
      parity ^= 1u;
    }
  }

  // Poll n tagged words into dst (fp32); all consumer threads take part.
  __device__ __forceinline__ void wait_words(const unsigned long long* src, int n, uint32_t want, float* dst) {
    for (int k0 = tid; k0 < n; k0 += 4 * kConsumers) {
      unsigned long long w[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int k = k0 + u * kConsumers;
        w[u] = k < n ? ld_tag(src + k) : 0ull;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int k = k0 + u * kConsumers;
        if (k >= n) break;
        if ((uint32_t)(w[u] >> 32) != want && !quit) {
          unsigned long long t0 = 0;
          int spins = 0;
          do {
            __nanosleep(32);
            w[u] = ld_tag(src + k);
            if ((++spins & 255) == 0) {
              if (t0 == 0) t0 = now_ns();
              if (aborted(p.abort_flag) || now_ns() - t0 > p.wait_ns) {
                if (!aborted(p.abort_flag)) raise_timeout(p);
                quit = true;
                break;
              }
            }
          } while ((uint32_t)(w[u] >> 32) != want);
        }
        dst[k] = __uint_as_float((uint32_t)w[u]);
      }
    }
  }

  // Gains of an RMSNorm, element tid + 256 j in register j (H <= 2048),
  // fetched before the wait for the activations so their latency overlaps it.
  __device__ __forceinline__ void load_gains(const __nv_bfloat16* g, float (&gr)[8]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int k = tid + kConsumers * j;
      gr[j] = k < p.H ? __bfloat162float(g[k]) : 0.f;
    }
  }

  // RMSNorm of the B rows of hs into xs with the preloaded gains.
  __device__ __forceinline__ void rmsnorm_rows(const float (&gr)[8]) {
    const int H = p.H;
    for (int b = 0; b < p.B; ++b) {
      float ss = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int k = tid + kConsumers * j;
        if (k < H) {
          const float v = hs[b * H + k];
          ss += v * v;
        }
      }
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) at[warp] = ss;
      consumer_sync();
      float tot = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) tot += at[w];
      const float inv = rsqrtf(tot / (float)H + p.eps);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int k = tid + kConsumers * j;
        if (k < H) xs[b * H + k] = hs[b * H + k] * inv * gr[j];
      }
      consumer_sync();
    }
  }

  __device__ __forceinline__ void phase_begin(int ph, int layer) {
    // Warps may still be on the previous phase's chunks (they read xs/hs).
    quit = consumer_sync_or(quit);
    if (quit) return;
    if (ph == kGU) tr(layer, 10);
    if (ph == kDown) tr(layer, 11);
    const int slot_layer = ph == kLM ? p.L : layer;
    if (ph == kQKV || ph == kO || ph == kLM) tr(slot_layer, ph == kO ? 3 : 0);
    const int H = p.H;
    const LayerDev& Lw = layers_s(p)[layer];
    float gr[8];
    switch (ph) {
      case kQKV:
        load_gains(Lw.attn_norm, gr);
        if (layer == p.l0) {
          for (int b = 0; b < p.B; ++b) {
            if (p.h_in) {
              for (int k = tid; k < H; k += kConsumers) hs[b * H + k] = p.h_in[b * H + k];
            } else {
              int t = p.tokens[b];
              if (t < 0 || t >= p.V) {
                if (tid == 0) atomicCAS(p.err, 0, kErrToken);
                t = 0;
              }
              for (int k = tid; k < H; k += kConsumers)
                hs[b * H + k] = __bfloat162float(p.embed[(size_t)t * H + k]);
            }
          }
          consumer_sync();
          if (p.capture && cta == 0)
            for (int b = 0; b < p.B; ++b)
              for (int k = tid; k < H; k += kConsumers)
                p.capture[((size_t)layer * p.capture_stride + b) * H + k] = hs[b * H + k];
        } else {
          wait_words(p.xh1, p.B * H, tag(layer - 1, 5), hs);
          quit = consumer_sync_or(quit);
          if (quit) return;
        }
        tr(layer, 1);
        rmsnorm_rows(gr);
        break;
      case kO:
        wait_words(p.xo, p.B * p.nq * p.d, tag(layer, 2), xs);
        quit = consumer_sync_or(quit);
        tr(layer, 4);
        break;
      case kGU:
        load_gains(Lw.ffn_norm, gr);
        wait_words(p.xh0, p.B * H, tag(layer, 3), hs);
        quit = consumer_sync_or(quit);
        if (quit) return;
        tr(layer, 5);
        rmsnorm_rows(gr);
        break;
      case kDown:
        wait_words(p.xa, p.B * p.I, tag(layer, 4), xs);
        quit = consumer_sync_or(quit);
        tr(layer, 6);
        break;
      case kLM:
        load_gains(p.final_norm, gr);
        if (p.l1 > p.l0) {
          wait_words(p.xh1, p.B * H, tag(p.l1 - 1, 5), hs);
        } else {
          for (int k = tid; k < p.B * H; k += kConsumers) hs[k] = p.h_in[k];
        }
        quit = consumer_sync_or(quit);
        if (quit) return;
        tr(p.L, 1);
        rmsnorm_rows(gr);
        break;
    }
  }

  // A phase's weight chunks. Warp w takes row w / segs, segment w % segs of
  // every chunk (gate/up: rows [0, rows) gate, [rows, 2 rows) up), so its
  // k-range is fixed for the phase: its slice of the activations is loaded
  // into registers once (when it fits) and each chunk costs IT unrolled
  // 16-byte loads and independent FMA chains. Warps run their chunks
  // independently: a warp that holds a whole row finishes it itself; rows
  // split over several warps (or a gate/up pair) are summed in shared memory
  // and the last warp to add finishes the row.
  __device__ __forceinline__ void gemv_phase(int ph, int layer, int a, int b, int K, ChunkShape cs) {
    const bool q8 = Q8W && ph != kLM;
#define FS_GP(R)                                               \
  if (cs.rows == R) {                                          \
    if (q8) gemv_phase_t<NB, Q8W, R>(ph, layer, a, b, K, cs);  \
    else gemv_phase_t<NB, false, R>(ph, layer, a, b, K, cs);   \
    return;                                                    \
  }
    FS_GP(8) FS_GP(4) FS_GP(2) FS_GP(1)
#undef FS_GP
    if (lane == 0) atomicCAS(p.err, 0, kErrBounds);  // a row does not fit a stage
    quit = true;
  }

  // Sum of 8 per-lane values v[0..7] over the warp in 9 shuffles: each step
  // halves the values a lane keeps. Afterwards lane l holds the total of
  // value r(l) = 4*bit4(l) + 2*bit3(l) + bit2(l).
  __device__ __forceinline__ float reduce8(const float (&v)[8]) {
    const bool h16 = lane & 16, h8 = lane & 8, h4 = lane & 4;
    float a[4], c[2];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float keep = h16 ? v[r + 4] : v[r];
      const float send = h16 ? v[r] : v[r + 4];
      a[r] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const float keep = h8 ? a[r + 2] : a[r];
      const float send = h8 ? a[r] : a[r + 2];
      c[r] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    const float keep = h4 ? c[1] : c[0];
    const float send = h4 ? c[0] : c[1];
    float t = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    t += __shfl_xor_sync(0xffffffffu, t, 2);
    t += __shfl_xor_sync(0xffffffffu, t, 1);
    return t;
  }

  // A phase's weight chunks. Chunk i of the stream belongs to consumer warp
  // i % (consumer warps), which alone waits for it, computes all of its (up
  // to 8) rows (gate/up: 4 gate and 4 up rows) over the whole input axis and
  // releases it; consecutive chunks are worked on by different warps at the
  // same time. The loop walks the input axis in blocks of 256: per block a
  // lane loads its 8 activations once (per batch row) and uses them for all 8
  // rows, whose FMA chains interleave. The code is the same for every K.
  template <int NBT, bool Q8, int R>
  __device__ __forceinline__ void gemv_phase_t(int ph, int layer, int a, int b, int K, ChunkShape cs) {
    const bool pair = ph == kGU;
    const int rb = Q8 ? K : 2 * K;
    const int kb = lane * 8;
    const int my_r = ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
    for (int n = a; n < b && !quit;) {
      const int e = chunk_end(p, ph, n, b, cs);
      const int nr = e - n;
      if ((int)(i % kConsumerWarps) == warp) {
        const unsigned char* st = stage_wait();
        const __half* sbase = reinterpret_cast<const __half*>(st + kWeightBytes);
        // row r of the work (pairs: r < 4 gate of pair r, r >= 4 up of pair r-4)
        // The chunk's R rows (pairs: R gate rows in v[0..R), R up rows in
        // v[4..4+R)) are computed without branches; in a short last chunk the
        // missing rows repeat its last row (in bounds) and their sums are dropped.
        constexpr int NV = 8;
        int srow[NV];
        bool used[NV];
#pragma unroll
        for (int r = 0; r < NV; ++r) {
          const int pr = (r & 3) < R ? (r & 3) : 0;
          const int cr = pr < nr ? pr : nr - 1;
          if (R == 8) {
            srow[r] = r < nr ? r : nr - 1;
            used[r] = true;
          } else if (pair) {
            srow[r] = r < 4 ? cr : cs.rows + cr;
            used[r] = (r & 3) < R;
          } else {
            srow[r] = r < R ? (r < nr ? r : nr - 1) : 0;
            used[r] = r < R;
          }
        }
        float acc[NV][NBT];
#pragma unroll
        for (int r = 0; r < NV; ++r)
#pragma unroll
          for (int bb = 0; bb < NBT; ++bb) acc[r][bb] = 0.f;
#pragma unroll 1
        for (int k0 = kb; k0 < K; k0 += 256) {
          float x8[NBT][8];
#pragma unroll
          for (int bb = 0; bb < NBT; ++bb) {
            if (bb < p.B) {
              const float4 a0 = *reinterpret_cast<const float4*>(xs + bb * K + k0);
              const float4 a1 = *reinterpret_cast<const float4*>(xs + bb * K + k0 + 4);
              x8[bb][0] = a0.x; x8[bb][1] = a0.y; x8[bb][2] = a0.z; x8[bb][3] = a0.w;
              x8[bb][4] = a1.x; x8[bb][5] = a1.y; x8[bb][6] = a1.z; x8[bb][7] = a1.w;
            } else {
#pragma unroll
              for (int q = 0; q < 8; ++q) x8[bb][q] = 0.f;
            }
          }
#pragma unroll
          for (int r = 0; r < NV; ++r) {
            if (!used[r]) continue;  // compile-time for a given R and phase kind
            float w[8];
            if (!Q8) {
              const uint4 u = *reinterpret_cast<const uint4*>(st + srow[r] * rb + k0 * 2);
              w[0] = lo16(u.x); w[1] = hi16(u.x); w[2] = lo16(u.y); w[3] = hi16(u.y);
              w[4] = lo16(u.z); w[5] = hi16(u.z); w[6] = lo16(u.w); w[7] = hi16(u.w);
#pragma unroll
              for (int bb = 0; bb < NBT; ++bb)
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[r][bb] = fmaf(w[q], x8[bb][q], acc[r][bb]);
            } else {
              // the lane's 8 codes share one block scale: dot the codes, scale once
              const uint2 u = *reinterpret_cast<const uint2*>(st + srow[r] * rb + k0);
              const float sc = __half2float(sbase[srow[r] * (K / 32) + k0 / 32]);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                w[q] = (float)(int8_t)((u.x >> (8 * q)) & 0xff);
                w[4 + q] = (float)(int8_t)((u.y >> (8 * q)) & 0xff);
              }
#pragma unroll
              for (int bb = 0; bb < NBT; ++bb) {
                float t = 0.f;
#pragma unroll
                for (int q = 0; q < 8; ++q) t = fmaf(w[q], x8[bb][q], t);
                acc[r][bb] = fmaf(sc, t, acc[r][bb]);
              }
            }
          }
        }
        stage_release();
        float tot[NBT], up[NBT];
#pragma unroll
        for (int bb = 0; bb < NBT; ++bb) {
          float col[8];
#pragma unroll
          for (int r = 0; r < 8; ++r) col[r] = acc[r][bb];
          tot[bb] = reduce8(col);
          up[bb] = pair ? __shfl_xor_sync(0xffffffffu, tot[bb], 16) : 0.f;
        }
        const bool mine = (lane & 3) == 0 && (pair ? my_r < 4 : true) && my_r < nr && !quit;
        if (mine) {
#pragma unroll
          for (int bb = 0; bb < NBT; ++bb)
            if (bb < p.B) epilogue(ph, layer, n + my_r, bb, tot[bb], up[bb]);
        }
      }
      advance();
      n = e;
    }
    if (p.trace && tid == 0 && (ph == kQKV || ph == kLM))
      p.trace[((size_t)cta * (p.L + 1) + (ph == kLM ? p.L : layer)) * 16 + (ph == kLM ? 6 : 8)] =
          clock64();
  }

  // Output of row n for batch row b (y = the dot product; u = the up row's
  // for a gate/up pair).
  __device__ __forceinline__ void epilogue(int ph, int layer, int n, int b, float y, float u) {
    switch (ph) {
      case kQKV:
        if (layer != p.withhold_layer)
          st_tag(p.xq + (size_t)b * (p.nq + 2 * p.nkv) * p.d + n, y, tag(layer, 1));
        break;
      case kO:
        st_tag(p.xh0 + (size_t)b * p.H + n, hs[b * p.H + n] + y, tag(layer, 3));
        break;
      case kGU:
        st_tag(p.xa + (size_t)b * p.I + n, y / (1.f + expf(-y)) * u, tag(layer, 4));
        break;
      case kDown: {
        const float h = hs[b * p.H + n] + y;
        st_tag(p.xh1 + (size_t)b * p.H + n, h, tag(layer, 5));
        if (p.capture) p.capture[((size_t)(layer + 1) * p.capture_stride + b) * p.H + n] = h;
        if (p.h_out && layer == p.l1 - 1) p.h_out[(size_t)b * p.H + n] = h;
        break;
      }
      case kLM: {
        if (p.logits) p.logits[(size_t)b * p.V + n] = y;
        if (isfinite(y)) {
          const uint32_t uu = (y == 0.f) ? 0u : __float_as_uint(y);  // -0 ranks as +0
          const uint32_t ord = (uu & 0x80000000u) ? ~uu : (uu | 0x80000000u);
          const unsigned long long key =
              ((unsigned long long)ord << 32) | (0xffffffffu - (uint32_t)n);
#pragma unroll
          for (int bb = 0; bb < kMaxB; ++bb)
            if (bb == b && key > wbest[bb]) wbest[bb] = key;
        }
        break;
      }
    }
  }

  // ---- attention ---------------------------------------------------------
  // Scratch (floats): q [rep][d] | knew [d] | vnew [d] | merge m,l [12][rep][2] | O [12][rep][d]
  // (a state per consumer warp, then the current position's key) | q fragments [512 words]
  __device__ float* q_s() { return at + 16; }
  __device__ float* k_s() { return q_s() + (p.nq / p.nkv) * p.d; }
  __device__ float* v_s() { return k_s() + p.d; }
  __device__ float* ml_s() { return v_s() + p.d; }
  __device__ float* acc_s() { return ml_s() + (kConsumerWarps + 1) * (p.nq / p.nkv) * 2; }
  __device__ uint32_t* qf_s() {  // q's B fragments [8 steps][2][32 lanes]
    return reinterpret_cast<uint32_t*>(acc_s() + (kConsumerWarps + 1) * (p.nq / p.nkv) * p.d);
  }

  // Per-lane constants of a head's RMSNorm + RoPE: gains of the lane's
  // elements of both halves and cos/sin at pos. Loaded before the wait for the
  // head's values, so their latency overlaps it.
  struct HeadConst {
    float g_lo[2], g_hi[2];
    float2 cs[2];
  };
  __device__ __forceinline__ void head_const(const __nv_bfloat16* gain, int pos, HeadConst& hc) {
    const int d = p.d, half = d / 2, E = d / 64;
    const float2* rp = p.rope + (size_t)pos * half;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int i = lane * E + e;
      const bool ok = e < E;
      hc.g_lo[e] = ok ? __bfloat162float(gain[i]) : 0.f;
      hc.g_hi[e] = ok ? __bfloat162float(gain[half + i]) : 0.f;
      hc.cs[e] = ok ? rp[i] : make_float2(0.f, 0.f);
    }
  }

  // RMSNorm over one head in a warp + rotate-half RoPE, in place.
  __device__ __forceinline__ void head_norm_rope(float* x, const HeadConst& hc) {
    const int d = p.d, half = d / 2;
    const int E = d / 64;  // elements per lane per half
    float lo[2] = {0.f, 0.f}, hi[2] = {0.f, 0.f}, ss = 0.f;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      if (e < E) {
        lo[e] = x[lane * E + e];
        hi[e] = x[half + lane * E + e];
        ss += lo[e] * lo[e] + hi[e] * hi[e];
      }
    }
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = rsqrtf(ss / (float)d + p.eps);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      if (e >= E) break;
      const int i = lane * E + e;
      const float a = lo[e] * inv * hc.g_lo[e];
      const float c = hi[e] * inv * hc.g_hi[e];
      x[i] = a * hc.cs[e].x - c * hc.cs[e].y;
      x[half + i] = c * hc.cs[e].x + a * hc.cs[e].y;
    }
  }

  __device__ __forceinline__ void attn_begin(int layer, int, const Item& x) {
    // The QKV chunks before this end on no barrier: decide quit CTA-wide first.
    quit = consumer_sync_or(quit);
    if (quit) return;
    tr(layer, 12);
    const int d = p.d, rep = p.nq / p.nkv, qd = p.nq * d, kvd = p.nkv * d;
    const unsigned long long* row = p.xq + (size_t)x.b * (qd + 2 * kvd);
    const uint32_t t1 = tag(layer, 1);
    const LayerDev& Lw = layers_s(p)[layer];
    const int pos = p.pos[x.b];
    HeadConst hc;
    if (warp < rep) head_const(Lw.q_norm, pos, hc);
    if (x.owner && warp == rep) head_const(Lw.k_norm, pos, hc);
    wait_words(row + x.g * rep * d, rep * d, t1, q_s());
    if (x.owner) {
      wait_words(row + qd + x.g * d, d, t1, k_s());
      wait_words(row + qd + kvd + x.g * d, d, t1, v_s());
    }
    quit = consumer_sync_or(quit);
    if (quit) return;
    tr(layer, 2);
    if (warp < rep) head_norm_rope(q_s() + warp * d, hc);
    if (x.owner && warp == rep) {
      head_norm_rope(k_s(), hc);
      const size_t off = kv_off(p, layer, x.b, pos, x.g);
      for (int i2 = lane; i2 < d; i2 += 32) {
        const __nv_bfloat16 kb = __float2bfloat16_rn(k_s()[i2]);
        const __nv_bfloat16 vb = __float2bfloat16_rn(v_s()[i2]);
        p.kv.k[off + i2] = kb;
        p.kv.v[off + i2] = vb;
        k_s()[i2] = __bfloat162float(kb);
        v_s()[i2] = __bfloat162float(vb);
      }
    }
    consumer_sync();
    tr(layer, 13);
    // q as the B operand of S = K q^T: column g = lane / 4 holds head g / 2,
    // term g % 2 (bf16 hi, then the lo remainder) of the scaled q; columns past
    // 2 * rep are zero. k-step kk covers dims 16 kk .. 16 kk + 15.
    // Built once per CTA into a table (word (kk, hf, lane)), then loaded by
    // every warp.
    const float scale = 1.f / sqrtf((float)d);
    uint32_t* qf = qf_s();
    for (int w = tid; w < 8 * 2 * 32; w += kConsumers) {
      const int kk = w >> 6, hf = (w >> 5) & 1, ln = w & 31, g = ln >> 2, t4 = ln & 3;
      uint32_t v = 0u;
      if (kk * 16 < d && g < 2 * rep) {
        const float* qh = q_s() + (g >> 1) * d + kk * 16 + hf * 8 + 2 * t4;
        v = bf16_term(qh[0] * scale, g & 1) | (bf16_term(qh[1] * scale, g & 1) << 16);
      }
      qf[w] = v;
    }
    consumer_sync();
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) qb[kk][hf] = qf[(kk * 2 + hf) * 32 + lane];
    mh = -INFINITY;
    lh = 0.f;
#pragma unroll
    for (int dt = 0; dt < 8; ++dt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[dt][e] = 0.f;
  }

  // One owner warp attends a whole KV chunk on the tensor cores and folds it
  // into its online-softmax state, 32 keys at a time. The chunk's K and V
  // tiles were loaded by TMA with the 128-byte swizzle: rows of 128 bytes
  // (64 dims), 16-byte unit u of row r stored at u ^ (r % 8), one block of
  // kpc rows per 64 dims. S = K q^T per 16 keys: A = 16 keys x 16 dims
  // (ldmatrix), B = q (hi / lo terms of both heads). Lane (g, t) = (lane / 4,
  // lane % 4) then holds the scores of keys g, g + 8, g + 16, g + 24 for head
  // t (t < rep). P V: A = V^T (ldmatrix.trans), B = P (hi / lo terms),
  // accumulated into O^T per 16-dim tile; the lane's columns 2t, 2t + 1
  // belong to head t.
  __device__ __forceinline__ void attend_chunk(const unsigned char* st, int nk) {
    const int d = p.d, rep = p.nq / p.nkv;
    const int nd = d >> 4;                         // 16-dim steps
    const uint32_t cbs = keys_per_chunk(d) * 128;  // bytes per 64-dim block of a tile
    const uint32_t kb = su32(st), vb = kb + kWeightBytes / 2;
    const int g = lane >> 2, t4 = lane & 3, mi = lane >> 3, rr = lane & 7;
    const int hn = g >> 1;  // head of this lane's B column
    const bool col_ok = g < 2 * rep, lo = g & 1, hv = t4 < rep;
    for (int kb0 = 0; kb0 < nk; kb0 += 32) {
      float sa[2][4], sb[2][4];  // per 16-key half: two accumulation chains
#pragma unroll
      for (int hf = 0; hf < 2; ++hf)
#pragma unroll
        for (int e = 0; e < 4; ++e) sa[hf][e] = sb[hf][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        if (kk < nd) {
          const int dim = kk * 16 + (mi >> 1) * 8;
          const uint32_t du = (uint32_t)(dim >> 6) * cbs, un = (dim & 63) >> 3;
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const int ka = kb0 + hf * 16 + (mi & 1) * 8 + rr;  // key row addressed (A = K)
            uint32_t a[4];
            ldsm_x4(kb + du + ka * 128 + ((un ^ (ka & 7)) << 4), a);
            if (kk & 1)
              mma_bf16(sb[hf], a, qb[kk][0], qb[kk][1]);
            else
              mma_bf16(sa[hf], a, qb[kk][0], qb[kk][1]);
          }
        }
      }
      float x[4];  // keys kb0 + g + 8 q
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int hf = q >> 1, e = (q & 1) * 2;
        const bool ok = hv && kb0 + g + 8 * q < nk;
        x[q] = ok ? (sa[hf][e] + sb[hf][e]) + (sa[hf][e + 1] + sb[hf][e + 1]) : -INFINITY;
      }
      float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
#pragma unroll
      for (int o2 = 4; o2 < 32; o2 <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
      const float mn = fmaxf(mh, mx);
      const float alpha = (mn == -INFINITY) ? 1.f : expf(mh - mn);
      float pr[4], sm = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        pr[q] = x[q] == -INFINITY ? 0.f : expf(x[q] - mn);
        sm += pr[q];
      }
#pragma unroll
      for (int o2 = 4; o2 < 32; o2 <<= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o2);
      lh = lh * alpha + sm;
      mh = mn;
#pragma unroll
      for (int dt = 0; dt < 8; ++dt)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[dt][e] *= alpha;
      // B = P per 16-key half: column g is head hn, term g % 2; keys 2t, 2t + 1
      // (b0) and 2t + 8, 2t + 9 (b1). Key k's probability for head hn sits in
      // lane (k % 8) * 4 + hn, value pr[k / 8].
      uint32_t pb[2][2];
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const float q00 = __shfl_sync(0xffffffffu, pr[2 * hf], (2 * t4) * 4 + hn);
        const float q01 = __shfl_sync(0xffffffffu, pr[2 * hf], (2 * t4 + 1) * 4 + hn);
        const float q10 = __shfl_sync(0xffffffffu, pr[2 * hf + 1], (2 * t4) * 4 + hn);
        const float q11 = __shfl_sync(0xffffffffu, pr[2 * hf + 1], (2 * t4 + 1) * 4 + hn);
        pb[hf][0] = col_ok ? bf16_term(q00, lo) | (bf16_term(q01, lo) << 16) : 0u;
        pb[hf][1] = col_ok ? bf16_term(q10, lo) | (bf16_term(q11, lo) << 16) : 0u;
      }
#pragma unroll
      for (int dt = 0; dt < 8; ++dt) {
        if (dt < nd) {
          const int dim = dt * 16 + (mi & 1) * 8;
          const uint32_t du = (uint32_t)(dim >> 6) * cbs, un = (dim & 63) >> 3;
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const int kv_ = kb0 + hf * 16 + (mi >> 1) * 8 + rr;  // key row (A = V^T)
            uint32_t a[4];
            ldsm_x4_t(vb + du + kv_ * 128 + ((un ^ (kv_ & 7)) << 4), a);
            mma_bf16(o[dt], a, pb[hf][0], pb[hf][1]);
          }
        }
      }
    }
  }

  // A KV chunk of the item, owner mode like the weight chunks: chunk i is
  // attended by warp i % (consumer warps) alone, which then releases it; the
  // warps' states are merged once, in attn_end.
  __device__ __forceinline__ void kv(int, const Item&, int, int nk) {
    if ((int)(i % kConsumerWarps) == warp) {
      const unsigned char* st = stage_wait();
      if (!__any_sync(0xffffffffu, quit)) attend_chunk(st, nk);
      stage_release();
    }
    advance();
  }

  __device__ __forceinline__ void attn_end(int layer, int, const Item& x) {
    // No early exit before the first barrier: threads may disagree on quit here.
    tr(layer, 14);
    const int d = p.d, rep = p.nq / p.nkv;
    constexpr int NSL = kConsumerWarps + 1;  // states: one per warp, then the new key
    float* ml = ml_s();
    float* ac = acc_s();
    // this warp's state: lanes (g, t < rep) hold head t's columns of O^T
    {
      const int g = lane >> 2, t4 = lane & 3;
      if (t4 < rep) {
        if (g == 0) {
          ml[(warp * rep + t4) * 2] = mh;
          ml[(warp * rep + t4) * 2 + 1] = lh;
        }
        float* a = ac + (warp * rep + t4) * d;
#pragma unroll
        for (int dt = 0; dt < 8; ++dt) {
          if (dt * 16 < d) {
            a[dt * 16 + g] = o[dt][0] + o[dt][1];
            a[dt * 16 + g + 8] = o[dt][2] + o[dt][3];
          }
        }
      }
    }
    // the last state: the current position's key, in the item that holds it
    if (warp == 0) {
      const float scale = 1.f / sqrtf((float)d);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (h >= rep) break;
        float sh = 0.f;
        for (int c = lane; c < d; c += 32) sh = fmaf(q_s()[h * d + c] * scale, k_s()[c], sh);
        for (int o2 = 16; o2 > 0; o2 >>= 1) sh += __shfl_xor_sync(0xffffffffu, sh, o2);
        if (lane == 0) {
          ml[(kConsumerWarps * rep + h) * 2] = x.owner ? sh : -INFINITY;
          ml[(kConsumerWarps * rep + h) * 2 + 1] = x.owner ? 1.f : 0.f;
        }
        for (int c = lane; c < d; c += 32)
          ac[(kConsumerWarps * rep + h) * d + c] = x.owner ? v_s()[c] : 0.f;
      }
    }
    quit = consumer_sync_or(quit);
    if (quit) return;
    const int ns = p.n_splits;
    const uint32_t t2 = tag(layer, 2);
    // merge the warps: first each warp's factor exp(m_w - M) per head (q's
    // space is free now), then one thread per (head, dim)
    float* fq = q_s();  // [state][rep] factors, then [rep] maxima
    if (tid < NSL * rep) {
      const int h = tid / NSL, w = tid - h * NSL;
      float M = -INFINITY;
      for (int w2 = 0; w2 < NSL; ++w2) M = fmaxf(M, ml[(w2 * rep + h) * 2]);
      const float mw = ml[(w * rep + h) * 2];
      fq[w * rep + h] = (mw == -INFINITY) ? 0.f : expf(mw - M);
      if (w == 0) fq[NSL * rep + h] = M;
    }
    consumer_sync();
    for (int t = tid; t < rep * d; t += kConsumers) {
      const int h = t / d, c = t % d;
      const float M = fq[NSL * rep + h];
      float L = 0.f, O = 0.f;
      for (int w = 0; w < NSL; ++w) {
        const float f = fq[w * rep + h];
        L = fmaf(ml[(w * rep + h) * 2 + 1], f, L);
        O = fmaf(ac[(w * rep + h) * d + c], f, O);
      }
      const int qh = x.g * rep + h;
      if (ns == 1) {
        st_tag(p.xo + (size_t)x.b * p.nq * d + qh * d + c, O / L, t2);
      } else {
        float* pp = p.part + ((((size_t)x.b * p.nkv + x.g) * ns + x.s) * rep + h) * (d + 2);
        if (c == 0) {
          pp[0] = M;
          pp[1] = L;
        }
        pp[2 + c] = O;
      }
    }
    tr(layer, 15);
    if (ns > 1) {
      __threadfence();
      consumer_sync();
      if (tid == 0) {
        unsigned int* cnt = p.split_cnt + x.b * p.nkv + x.g;
        const unsigned int old = atomicAdd(cnt, 1u);
        *flag = (old == (unsigned int)ns - 1);
        if (*flag) atomicExch(cnt, 0u);
      }
      consumer_sync();
      if (*flag) {
        __threadfence();
        for (int t = tid; t < rep * d; t += kConsumers) {
          const int h = t / d, c = t % d;
          const float* base = p.part + (((size_t)x.b * p.nkv + x.g) * ns * rep + h) * (d + 2);
          float M = -INFINITY;
          for (int s = 0; s < ns; ++s) M = fmaxf(M, __ldcg(base + (size_t)s * rep * (d + 2)));
          float L = 0.f, O = 0.f;
          for (int s = 0; s < ns; ++s) {
            const float* q = base + (size_t)s * rep * (d + 2);
            const float ms = __ldcg(q);
            const float f = (ms == -INFINITY) ? 0.f : expf(ms - M);
            L += __ldcg(q + 1) * f;
            O += __ldcg(q + 2 + c) * f;
          }
          st_tag(p.xo + (size_t)x.b * p.nq * d + (x.g * rep + h) * d + c, O / L, t2);
        }
      }
    }
    quit = consumer_sync_or(quit);
    tr(layer, 9);
  }

  __device__ void end_layer() {
    quit = consumer_sync_or(quit);
    tr(cur_layer, 7);
    ++cur_layer;
  }
  int cur_layer = 0;

  // End of the step: fold this CTA's greedy keys; the last CTA writes ids.
  __device__ __forceinline__ void finish_head() {
    if (!p.run_head) return;
#pragma unroll
    for (int bb = 0; bb < kMaxB; ++bb) {
      unsigned long long k = wbest[bb];
      for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long other = __shfl_xor_sync(0xffffffffu, k, o);
        k = other > k ? other : k;
      }
      if (lane == 0 && bb < p.B && k) atomicMax(best + bb, k);
    }
    quit = consumer_sync_or(quit);
    tr(p.L, 7);
    if (tid < p.B && !quit) atomicMax(p.am_key + tid, best[tid]);
    __threadfence();
    consumer_sync();
    if (tid == 0) {
      const unsigned int old = atomicAdd(p.am_cnt, 1u);
      *flag = (old == (unsigned int)G - 1);
    }
    consumer_sync();
    if (*flag) {
      __threadfence();
      if (tid < p.B) {
        const unsigned long long key = atomicExch(p.am_key + tid, 0ull);
        int id = 0;
        if (key == 0ull) {
          atomicCAS(p.err, 0, kErrBounds);
        } else {
          id = (int)(0xffffffffu - (uint32_t)(key & 0xffffffffu));
        }
        if (p.argmax) p.argmax[tid] = id;
      }
      if (tid == 0) atomicExch(p.am_cnt, 0u);
    }
  }
};

template <int NB, bool Q8W>
__global__ void __launch_bounds__(kThreads, 1)
    decode_mega_kernel(const __grid_constant__ Params p, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v) {
  extern __shared__ __align__(1024) unsigned char smem[];
  Ring ring;
  ring.stages = smem;
  ring.n = p.n_stages;
  ring.full = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  ring.empty = ring.full + kMaxStages;
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.n_stages; ++s) {
      mbar_init(&ring.full[s], 1);
      mbar_init(&ring.empty[s], 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    unsigned long long* best = reinterpret_cast<unsigned long long*>(smem + p.off_misc);
    for (int b = 0; b < kMaxB; ++b) best[b] = 0ull;
  }
  {
    const unsigned* src = reinterpret_cast<const unsigned*>(p.layers);
    unsigned* dst = reinterpret_cast<unsigned*>(smem + p.off_tab);
    const int words = p.L * (int)sizeof(LayerDev) / 4;
    for (int k = threadIdx.x; k < words; k += blockDim.x) dst[k] = src[k];
    if (p.bt_in_smem) {
      int32_t* bt = reinterpret_cast<int32_t*>(smem + p.off_tab + (size_t)p.L * sizeof(LayerDev));
      const int pps = p.kv.pages_per_seq;
      for (int k = threadIdx.x; k < p.B * pps; k += blockDim.x)
        bt[k] = p.kv.block_table[(size_t)p.seq[k / pps] * pps + k % pps];
    }
  }
  unsigned long long* trow =
      p.trace ? p.trace + ((size_t)blockIdx.x * (p.L + 1) + p.L) * 16 : nullptr;
  if (trow && threadIdx.x == 0) {  // time base: (%globaltimer, clock64) at start and end
    trow[12] = now_ns();
    trow[13] = clock64();
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  if (warp == kConsumerWarps) {
    // producer warp: one lane issues, the others go straight to the end
    if ((threadIdx.x & 31) == 0) {
      Producer pr(p, ring, &tm_k, &tm_v);
      walk(p, blockIdx.x, gridDim.x, pr);
      if (p.trace) p.trace[((size_t)blockIdx.x * (p.L + 1) + p.L) * 16 + 3] = clock64();
      reinterpret_cast<volatile unsigned int*>(smem + p.off_misc + 8 * kMaxB + 8)[0] = pr.i;
    }
  } else {
    Consumer<NB, Q8W> cs(p, ring, smem);
    walk(p, blockIdx.x, gridDim.x, cs);
    cs.finish_head();
    if (threadIdx.x == 0)
      reinterpret_cast<volatile unsigned int*>(smem + p.off_misc + 8 * kMaxB + 12)[0] = cs.i;
  }
  __syncthreads();
  // Drain: a stage issued but never consumed (after an abort) must land
  // before the CTA's shared memory is released.
  if (threadIdx.x == 0) {
    const unsigned int issued =
        reinterpret_cast<volatile unsigned int*>(smem + p.off_misc + 8 * kMaxB + 8)[0];
    const unsigned int used =
        reinterpret_cast<volatile unsigned int*>(smem + p.off_misc + 8 * kMaxB + 12)[0];
    const unsigned int first =
        issued > (unsigned int)ring.n && issued - ring.n > used ? issued - ring.n : used;
    for (unsigned int k = first; k < issued; ++k) {
      const unsigned long long t0 = now_ns();
      while (!mbar_test(&ring.full[k % ring.n], (k / ring.n) & 1))
        if (now_ns() - t0 > 10000000ull) break;  // 10 ms
    }
    if (trow) {
      trow[14] = now_ns();
      trow[15] = clock64();
    }
  }
}

}  // namespace mega

// ---------------------------------------------------------------------------
// Host side

namespace {

struct MegaState {
  unsigned long long *xq = nullptr, *xo = nullptr, *xh0 = nullptr, *xh1 = nullptr, *xa = nullptr;
  float* part = nullptr;
  unsigned int* split_cnt = nullptr;
  unsigned long long* am_key = nullptr;
  unsigned int* am_cnt = nullptr;
  int* abort_flag = nullptr;
  LayerDev* layers = nullptr;
  uint32_t next_tag = 1;
  int max_splits = 0;
  int sms = 0;
  bool eligible = false;
  unsigned long long wait_ns = 1000000000ull;
  int withhold = -1;
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Keys per attention item of a decode step: one KV chunk per consumer warp,
// all attended at once (the items of a kv head are merged by the last one to
// finish).
#ifndef FS_MEGA_LONG_CHUNKS
#define FS_MEGA_LONG_CHUNKS 4
#endif
// A context that fits one item of a chunk per consumer warp takes one item per
// kv head (no merge of splits); a longer one is cut into items of
// FS_MEGA_LONG_CHUNKS chunks, spread over more CTAs (each CTA then streams
// fewer KV bytes per block).
int keys_per_split(int d, int context) {
  const int one = mega::kConsumerWarps * mega::keys_per_chunk(d);
  return context <= one ? one : FS_MEGA_LONG_CHUNKS * mega::keys_per_chunk(d);
}

}  // namespace

bool mega_shape_ok(const fs_model* m) {
  const Shape& s = m->s;
  const int rep = s.nq / s.nkv;
  if (rep > 2 || (s.d != 64 && s.d != 128)) return false;
  if (s.V >= 0x7fffffff || s.H > 2048) return false;
  auto it_ok = [](int K) {
    if (K % 256) return false;
    const int it = K / 256;
    return it == 1 || it == 2 || it == 3 || it == 4 || it == 6 || it == 8 || it == 12;
  };
  const int Ks[3] = {s.H, s.q_dim(), s.I};
  for (int K : Ks)
    if (!it_ok(K)) return false;
  // every phase needs at least one whole row (pair) per stage
  if (mega::chunk_shape(s.I, m->q8, false).rows < 1 || mega::chunk_shape(s.H, m->q8, true).rows < 1 ||
      mega::chunk_shape(s.q_dim(), m->q8, false).rows < 1)
    return false;
  return true;
}

static void mega_free(MegaState* st) {
  void* bufs[] = {st->xq, st->xo, st->xh0, st->xh1, st->xa, st->part,
                  st->split_cnt, st->am_key, st->am_cnt, st->abort_flag, st->layers};
  for (void* b : bufs)
    if (b) cudaFree(b);
}

fs_status mega_init(fs_model* m) {
  MegaState* st = new MegaState();
  m->mega_extras = st;
  st->sms = m->num_sms;
  st->eligible = mega_shape_ok(m);
  if (!st->eligible) return FS_OK;
  const Shape& s = m->s;
  const int B = mega::kMaxB;
  const int rep = s.nq / s.nkv;
  st->max_splits = std::max(1, st->sms / s.nkv);
  auto alloc = [&](void** p, size_t bytes) {
    if (cudaMalloc(p, bytes) != cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    cudaMemset(*p, 0, bytes);
    return true;
  };
  const size_t w = sizeof(unsigned long long);
  bool ok = alloc((void**)&st->xq, (size_t)B * s.qkv_dim() * w) &&
            alloc((void**)&st->xo, (size_t)B * s.q_dim() * w) &&
            alloc((void**)&st->xh0, (size_t)B * s.H * w) &&
            alloc((void**)&st->xh1, (size_t)B * s.H * w) &&
            alloc((void**)&st->xa, (size_t)B * s.I * w) &&
            alloc((void**)&st->part,
                  (size_t)B * s.nkv * st->max_splits * rep * (s.d + 2) * sizeof(float)) &&
            alloc((void**)&st->split_cnt, (size_t)B * s.nkv * sizeof(unsigned int)) &&
            alloc((void**)&st->am_key, (size_t)B * w) &&
            alloc((void**)&st->am_cnt, 64) && alloc((void**)&st->abort_flag, 64) &&
            alloc((void**)&st->layers, (size_t)s.L * sizeof(LayerDev));
  if (!ok) {
    mega_free(st);
    delete st;
    m->mega_extras = nullptr;
    set_error("out of device memory for the decode exchange buffers");
    return FS_ERR_OOM;
  }
  cudaMemcpy(st->layers, m->layers.data(), (size_t)s.L * sizeof(LayerDev),
             cudaMemcpyHostToDevice);
  const void* kernels[4] = {(const void*)mega::decode_mega_kernel<1, false>,
                            (const void*)mega::decode_mega_kernel<1, true>,
                            (const void*)mega::decode_mega_kernel<4, false>,
                            (const void*)mega::decode_mega_kernel<4, true>};
  for (const void* k : kernels)
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
  return FS_OK;
}

void mega_release(fs_model* m) {
  MegaState* st = static_cast<MegaState*>(m->mega_extras);
  if (!st) return;
  mega_free(st);
  delete st;
  m->mega_extras = nullptr;
}

// Resets the exchange state after a step was aborted (device error seen).
void mega_reset(fs_model* m) {
  MegaState* st = static_cast<MegaState*>(m->mega_extras);
  if (!st || !st->eligible) return;
  cudaDeviceSynchronize();
  cudaMemset(st->split_cnt, 0, (size_t)mega::kMaxB * m->s.nkv * sizeof(unsigned int));
  cudaMemset(st->am_key, 0, (size_t)mega::kMaxB * sizeof(unsigned long long));
  cudaMemset(st->am_cnt, 0, 64);
  cudaMemset(st->abort_flag, 0, 64);
  st->next_tag += 1u << 20;  // every tag in flight is now stale
}

// Runs layers [l0, l1) (and the LM head if run_head) of one decode step for
// B <= 4 rows. Returns FS_ERR_UNSUPPORTED when the shape or batch is not
// covered or the ring would get fewer stages than consumer warps (the caller
// then uses the general path).
void mega_debug_wait(fs_model* m, unsigned long long wait_ns, int withhold_layer) {
  MegaState* st = static_cast<MegaState*>(m->mega_extras);
  if (!st) return;
  st->wait_ns = wait_ns;
  st->withhold = withhold_layer;
}

bool mega_eligible(const fs_model* m) {
  const MegaState* st = static_cast<const MegaState*>(m->mega_extras);
  return st && st->eligible;
}

fs_status decode_mega(fs_model* m, const fs_kv* kv, const RowMap& map, int B, const int32_t* tok,
                      const float* h_in, float* h_out, int l0, int l1, bool run_head,
                      float* logits, int32_t* argmax, cudaStream_t stream) {
  MegaState* st = static_cast<MegaState*>(m->mega_extras);
  if (!st || !st->eligible || B > mega::kMaxB || B < 1) return FS_ERR_UNSUPPORTED;
  const Shape& s = m->s;
  const int rep = s.nq / s.nkv;
  mega::Params p{};
  p.L = s.L; p.H = s.H; p.nq = s.nq; p.nkv = s.nkv; p.d = s.d; p.I = s.I; p.V = s.V;
  p.eps = s.eps;
  p.q8 = m->q8 ? 1 : 0;
  p.layers = st->layers;
  p.embed = m->embed;
  p.final_norm = m->final_norm;
  p.rope = m->rope;
  p.kv = kv_view(kv);
  p.B = B;
  int cmax = 1;
  for (int b = 0; b < B; ++b) {
    const RowInfo ri = map.get(b);
    p.seq[b] = ri.seq;
    p.pos[b] = ri.pos;
    cmax = std::max(cmax, ri.pos + 1);
  }
  p.tokens = tok;
  p.xq = st->xq; p.xo = st->xo; p.xh0 = st->xh0; p.xh1 = st->xh1; p.xa = st->xa;
  p.part = st->part;
  p.split_cnt = st->split_cnt;
  p.am_key = st->am_key;
  p.am_cnt = st->am_cnt;
  // at most one item per CTA
  const int kps = keys_per_split(s.d, cmax);
  int ns = (cmax + kps - 1) / kps;
  ns = std::max(1, std::min(ns, std::min(st->max_splits, st->sms / (B * s.nkv))));
  p.n_splits = ns;
  p.l0 = l0;
  p.l1 = l1;
  p.h_in = h_in;
  p.h_out = h_out;
  p.run_head = run_head ? 1 : 0;
  p.logits = logits;
  p.argmax = argmax;
  p.capture = m->capture;
  p.capture_stride = m->capture_max_rows;
  p.err = m->err;
  p.abort_flag = st->abort_flag;
  p.wait_ns = st->wait_ns;
  p.withhold_layer = st->withhold;
  st->withhold = -1;  // one-shot
  p.trace = m->trace;
  m->trace = nullptr;  // one-shot
  const uint32_t span = 5u * (uint32_t)(l1 - l0) + 2u;
  if (st->next_tag > 0xF0000000u) {
    // wrap: clear the tags so the numbering can restart
    cudaStreamSynchronize(stream);
    const size_t w = sizeof(unsigned long long);
    cudaMemsetAsync(st->xq, 0, (size_t)mega::kMaxB * s.qkv_dim() * w, stream);
    cudaMemsetAsync(st->xo, 0, (size_t)mega::kMaxB * s.q_dim() * w, stream);
    cudaMemsetAsync(st->xh0, 0, (size_t)mega::kMaxB * s.H * w, stream);
    cudaMemsetAsync(st->xh1, 0, (size_t)mega::kMaxB * s.H * w, stream);
    cudaMemsetAsync(st->xa, 0, (size_t)mega::kMaxB * s.I * w, stream);
    st->next_tag = 1;
  }
  p.tag0 = st->next_tag;
  st->next_tag += span;
  // shared memory carve-up
  const int maxK = std::max({s.H, s.q_dim(), s.I});
  size_t off = 0;
  const size_t fixed_hs = align_up((size_t)B * s.H * 4, 128);
  const size_t fixed_xs = align_up((size_t)B * maxK * 4, 128);
  const size_t attn = align_up((16 + rep * s.d + 2 * s.d + (mega::kConsumerWarps + 1) * rep * 2 +
                                (mega::kConsumerWarps + 1) * rep * s.d + 512) * 4, 128);
  const size_t bars = 2 * mega::kMaxStages * 8;
  const size_t misc = 128;
  const size_t bt_bytes = (size_t)B * kv->pages_per_seq * sizeof(int32_t);
  const bool bt_smem = bt_bytes <= 8192;
  const size_t tab = align_up((size_t)s.L * sizeof(LayerDev) + (bt_smem ? bt_bytes : 0), 128);
  const size_t fixed = fixed_hs + fixed_xs + attn + bars + misc + tab;
  const size_t budget = 232448;
  int n_stages = (int)((budget - fixed) / mega::kStageBytes);
  n_stages = std::min(n_stages, mega::kMaxStages);
  // Any ring of two or more stages is correct (see Consumer::stage_wait);
  // fewer stages only bound how far the weight stream runs ahead.
  // weight chunk i belongs to warp i mod 11, which tests the release of the
  // chunk a ring earlier before the chunk: unambiguous with a stage per warp
  if (n_stages < mega::kConsumerWarps) return FS_ERR_UNSUPPORTED;
  off = (size_t)n_stages * mega::kStageBytes;
  p.off_hs = (int)off; off += fixed_hs;
  p.off_xs = (int)off; off += fixed_xs;
  p.off_attn = (int)off; off += attn;
  p.off_bar = (int)off; off += bars;
  p.off_misc = (int)off; off += misc;
  p.off_tab = (int)off; off += tab;
  p.bt_in_smem = bt_smem ? 1 : 0;
  p.n_stages = n_stages;
  // the KV cache as [rows][d] bf16 for the attention items' TMA loads
  const long long kv_rows = (long long)s.L * kv->n_pages * s.nkv * kPage;
  if (kv_rows + 64 >= (1LL << 31)) return FS_ERR_UNSUPPORTED;
  CUtensorMap tm_k, tm_v;
  if (!make_tmap_16(&tm_k, kv->k, kv_rows, s.d, 32, true) ||
      !make_tmap_16(&tm_v, kv->v, kv_rows, s.d, 32, true))
    return FS_ERR_UNSUPPORTED;
  void* args[] = {&p, &tm_k, &tm_v};
  count_launches();
  const void* fn = B == 1 ? (m->q8 ? (const void*)mega::decode_mega_kernel<1, true>
                                    : (const void*)mega::decode_mega_kernel<1, false>)
                         : (m->q8 ? (const void*)mega::decode_mega_kernel<4, true>
                                  : (const void*)mega::decode_mega_kernel<4, false>);
  cudaError_t e = cudaLaunchCooperativeKernel(fn,
                                              dim3(st->sms), dim3(mega::kThreads), args, off,
                                              stream);
  if (e != cudaSuccess) {
    set_error(std::string("decode kernel launch failed: ") + cudaGetErrorString(e));
    return FS_ERR_CUDA;
  }
  return FS_OK;
}

}  // namespace fs
