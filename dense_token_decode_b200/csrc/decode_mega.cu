// Persistent decode forward: one cooperative launch runs every block and the
// LM head of one decode step for a batch of up to 4 sequences.
//
// Layout of the work. Each CTA (one per SM) owns a contiguous slice of the
// rows of every weight matrix. A producer warp streams the CTA's slices —
// QKV rows, the old K/V pages of the CTA's attention items, O rows, gate/up
// row pairs, down rows, per layer, then its rows of the tied embedding for
// the LM head — through a ring of shared-memory stages with cp.async.bulk.
// Weights do not depend on activations, so the producer runs ahead across
// phase and layer boundaries and HBM never waits for the dependency chain.
//
// Eight consumer warps compute. Activations move between CTAs as 64-bit
// words (fp32 value | 32-bit tag): a consumer polls the words it needs until
// their tag is the one of the current phase, so there is no grid barrier and
// no separate flag. Tags grow monotonically across steps; nothing is reset.
//
// Phases of block l (tag t_l,p): P1 RMSNorm + QKV rows -> xq; P2 attention
// items (b, kv head g, split s): q/k head RMSNorm + RoPE, append of the new
// K/V to the page, online-softmax attention over the split's keys, merge of
// splits by the last arriving item -> xo; P3 O rows + residual -> xh0;
// P4 RMSNorm + gate/up pairs + SwiGLU -> xa; P5 down rows + residual -> xh1.
// LM head: final RMSNorm, logits of the CTA's vocab rows, greedy key (value,
// lowest id) folded with a 64-bit atomicMax; the last CTA writes the ids.
//
// Every wait is bounded by %globaltimer; on timeout the CTA records
// kErrTimeout in the error word, stops waiting, drains its own bulk copies
// and returns.
#include <algorithm>

#include "runtime.h"

namespace fs {
namespace mega {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;  // + producer warp
constexpr int kMaxB = 4;
constexpr int kWeightBytes = 16384;             // weight bytes of one stage
constexpr int kStageBytes = kWeightBytes + 1024; // + Q8_0 scales
constexpr int kMaxStages = 16;
constexpr unsigned long long kTimeoutNs = 1000000000ull;  // 1 s per wait

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
  unsigned long long* trace;  // optional: %globaltimer stamps [G][L+1][8]
  int n_stages;
  // smem carve-up (bytes)
  int off_hs, off_xs, off_attn, off_red, off_bar, off_misc;
};

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

// ---------------------------------------------------------------------------
// Shapes of the chunk stream (identical in producer and consumers)

struct ChunkShape {
  int rows;  // weight rows per chunk (gate/up: pairs)
  int segs;  // warps per row
};

__host__ __device__ inline ChunkShape chunk_shape(int K, bool q8, bool pair) {
  const int row_bytes = q8 ? K : 2 * K;
  const int mult = pair ? 2 : 1;
  int rows = 8 / mult;
  while (rows > 1 && rows * mult * row_bytes > kWeightBytes) rows >>= 1;
  return ChunkShape{rows, kConsumerWarps / (rows * mult)};
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
  const LayerDev& Lw = p.layers[layer];
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

  __device__ Producer(const Params& pp, Ring rr) : p(pp), r(rr) { policy = evict_first_policy(); }
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
      if ((++spins & 1023) == 0) {
        if (t0 == 0) t0 = now_ns();
        if (aborted(p.abort_flag) || now_ns() - t0 > kTimeoutNs) {
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
      unsigned long long* t = p.trace + ((size_t)blockIdx.x * (p.L + 1) + p.L) * 8;
      if (!lm_started) t[2] = now_ns();
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
      const LayerDev& Lw = p.layers[layer];
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

  __device__ void kv(int layer, const Item& x, int j, int nk) {
    if (quit) return;
    const uint32_t bytes = 2u * nk * p.d * 2;
    unsigned char* st = acquire(bytes);
    if (!st) return;
    const size_t off = p.kv.offset(layer, p.seq[x.b], j, x.g);
    uint64_t* bar = &r.full[stage];
    bulk_load(st, p.kv.k + off, nk * p.d * 2, bar, policy);
    bulk_load(st + kWeightBytes / 2, p.kv.v + off, nk * p.d * 2, bar, policy);
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
  float* comb;  // [stages][8 rows][2][kMaxB] partial sums of split rows
  int* ccnt;    // [stages][8 rows] arrivals per split row
  float* at;    // attention scratch
  unsigned long long wbest = 0ull;  // lane b: this warp's greedy key of batch row b
  unsigned long long* best;  // [kMaxB] greedy keys of this CTA
  int* flag;
  unsigned int i = 0;  // chunks consumed
  int stage = 0;       // i % ring size
  uint32_t parity = 0; // (i / ring size) & 1
  bool quit = false;
  int tid, warp, lane;
  int G, cta;
  // attention state (per warp, registers)
  float qreg[2][4];
  float m[2], l[2], acc[2][4];

  __device__ Consumer(const Params& pp, Ring rr, unsigned char* sm) : p(pp), r(rr), smem(sm) {
    hs = reinterpret_cast<float*>(sm + p.off_hs);
    xs = reinterpret_cast<float*>(sm + p.off_xs);
    at = reinterpret_cast<float*>(sm + p.off_attn);
    comb = reinterpret_cast<float*>(sm + p.off_red);
    ccnt = reinterpret_cast<int*>(sm + p.off_red + kMaxStages * kConsumerWarps * 2 * kMaxB * 4);
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
    if (p.trace && tid == 0) p.trace[((size_t)cta * (p.L + 1) + layer) * 8 + k] = now_ns();
  }

  __device__ uint32_t tag(int layer, int ph) const {
    return p.tag0 + 5u * (uint32_t)(layer - p.l0) + (uint32_t)ph;
  }

  // Wait for the ring stage of the next chunk. On a timeout the thread sets
  // quit and carries on with whatever the stage holds until the next
  // reducing barrier makes the decision CTA-wide.
  __device__ const unsigned char* stage_wait() {
    const int s = stage;
    unsigned long long t0 = 0;
    int spins = 0;
    // Every lane observes the barrier itself (that is what makes the bulk
    // copy's bytes visible to it); the give-up decision is lane 0's, so the
    // warp stays converged for the shuffles that follow.
    while (true) {
      const bool ok = quit || mbar_test(&r.full[s], parity);
      if (__all_sync(0xffffffffu, ok)) break;
      if ((++spins & 1023) == 0) {
        int bad = 0;
        if (lane == 0) {
          if (t0 == 0) t0 = now_ns();
          bad = aborted(p.abort_flag) || now_ns() - t0 > kTimeoutNs;
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
            w[u] = ld_tag(src + k);
            if ((++spins & 255) == 0) {
              if (t0 == 0) t0 = now_ns();
              if (aborted(p.abort_flag) || now_ns() - t0 > kTimeoutNs) {
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

  // RMSNorm of the B rows of hs into xs with bf16 gains g.
  __device__ __forceinline__ void rmsnorm_rows(const __nv_bfloat16* g) {
    const int H = p.H;
    for (int b = 0; b < p.B; ++b) {
      float ss = 0.f;
      for (int k = tid; k < H; k += kConsumers) {
        const float v = hs[b * H + k];
        ss += v * v;
      }
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) at[warp] = ss;
      consumer_sync();
      float tot = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) tot += at[w];
      const float inv = rsqrtf(tot / (float)H + p.eps);
      for (int k = tid; k < H; k += kConsumers)
        xs[b * H + k] = hs[b * H + k] * inv * __bfloat162float(g[k]);
      consumer_sync();
    }
  }

  __device__ __forceinline__ void phase_begin(int ph, int layer) {
    // Warps may still be on the previous phase's chunks (they read xs/hs).
    quit = consumer_sync_or(quit);
    if (quit) return;
    const int slot_layer = ph == kLM ? p.L : layer;
    if (ph == kQKV || ph == kO || ph == kLM) tr(slot_layer, ph == kO ? 3 : 0);
    const int H = p.H;
    const LayerDev& Lw = p.layers[layer];
    switch (ph) {
      case kQKV:
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
        rmsnorm_rows(Lw.attn_norm);
        break;
      case kO:
        wait_words(p.xo, p.B * p.nq * p.d, tag(layer, 2), xs);
        quit = consumer_sync_or(quit);
        tr(layer, 4);
        break;
      case kGU:
        wait_words(p.xh0, p.B * H, tag(layer, 3), hs);
        quit = consumer_sync_or(quit);
        if (quit) return;
        tr(layer, 5);
        rmsnorm_rows(Lw.ffn_norm);
        break;
      case kDown:
        wait_words(p.xa, p.B * p.I, tag(layer, 4), xs);
        quit = consumer_sync_or(quit);
        tr(layer, 6);
        break;
      case kLM:
        if (p.l1 > p.l0) {
          wait_words(p.xh1, p.B * H, tag(p.l1 - 1, 5), hs);
        } else {
          for (int k = tid; k < p.B * H; k += kConsumers) hs[k] = p.h_in[k];
        }
        quit = consumer_sync_or(quit);
        if (quit) return;
        tr(p.L, 1);
        rmsnorm_rows(p.final_norm);
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
    const int it = (K / cs.segs) / 256;
    const bool q8 = Q8W && ph != kLM;
#define FS_GP(IT, NB)                                                     \
  if (it == IT) {                                                         \
    if (q8) gemv_phase_t<IT, NB, Q8W>(ph, layer, a, b, K, cs);            \
    else gemv_phase_t<IT, NB, false>(ph, layer, a, b, K, cs);             \
    return;                                                               \
  }
#define FS_GP_B(NB) FS_GP(1, NB) FS_GP(2, NB) FS_GP(3, NB) FS_GP(4, NB) FS_GP(6, NB) FS_GP(8, NB)
    FS_GP_B(NB)
#undef FS_GP_B
#undef FS_GP
    if (lane == 0) atomicCAS(p.err, 0, kErrBounds);  // unsupported chunk shape
    quit = true;
  }

  template <int IT, int NBT, bool Q8>
  __device__ __forceinline__ void gemv_phase_t(int ph, int layer, int a, int b, int K, ChunkShape cs) {
    constexpr bool XREG = NBT * IT * 8 <= 64;
    const bool pair = ph == kGU;
    const int rb = Q8 ? K : 2 * K;
    const int seg_len = K / cs.segs;
    const int ri = warp / cs.segs, seg = warp % cs.segs;
    const int mrow = pair ? (ri < cs.rows ? ri : ri - cs.rows) : ri;
    const int kb = seg * seg_len + lane * 8;  // this lane's first element; then +256 per j
    const int B = p.B;
    float xr[XREG ? NBT : 1][XREG ? IT : 1][8];
    if (XREG) {
#pragma unroll
      for (int bb = 0; bb < NBT; ++bb)
#pragma unroll
        for (int j = 0; j < IT; ++j) {
          const bool ok = bb < B;
          const float4 a0 = ok ? *reinterpret_cast<const float4*>(xs + bb * K + kb + 256 * j)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
          const float4 a1 = ok ? *reinterpret_cast<const float4*>(xs + bb * K + kb + 256 * j + 4)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
          xr[bb][j][0] = a0.x; xr[bb][j][1] = a0.y; xr[bb][j][2] = a0.z; xr[bb][j][3] = a0.w;
          xr[bb][j][4] = a1.x; xr[bb][j][5] = a1.y; xr[bb][j][6] = a1.z; xr[bb][j][7] = a1.w;
        }
    }
    for (int n = a; n < b && !quit;) {
      const int e = chunk_end(p, ph, n, b, cs);
      const int nr = e - n;
      const unsigned char* st = stage_wait();
      const bool valid = mrow < nr && !quit;
      float part[NBT][IT];
#pragma unroll
      for (int bb = 0; bb < NBT; ++bb)
#pragma unroll
        for (int j = 0; j < IT; ++j) part[bb][j] = 0.f;
      if (valid) {
        const unsigned char* row = st + ri * rb;
        float w[IT][8];
        if (!Q8) {
          uint4 u[IT];
#pragma unroll
          for (int j = 0; j < IT; ++j) u[j] = *reinterpret_cast<const uint4*>(row + (kb + 256 * j) * 2);
#pragma unroll
          for (int j = 0; j < IT; ++j) {
            w[j][0] = lo16(u[j].x); w[j][1] = hi16(u[j].x); w[j][2] = lo16(u[j].y); w[j][3] = hi16(u[j].y);
            w[j][4] = lo16(u[j].z); w[j][5] = hi16(u[j].z); w[j][6] = lo16(u[j].w); w[j][7] = hi16(u[j].w);
          }
        } else {
          uint2 u[IT];
          float sc[IT];
          const __half* srow = reinterpret_cast<const __half*>(st + kWeightBytes) + ri * (K / 32);
#pragma unroll
          for (int j = 0; j < IT; ++j) {
            u[j] = *reinterpret_cast<const uint2*>(row + kb + 256 * j);
            sc[j] = __half2float(srow[(kb + 256 * j) / 32]);
          }
#pragma unroll
          for (int j = 0; j < IT; ++j)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              w[j][q] = (float)(int8_t)((u[j].x >> (8 * q)) & 0xff) * sc[j];
              w[j][4 + q] = (float)(int8_t)((u[j].y >> (8 * q)) & 0xff) * sc[j];
            }
        }
#pragma unroll
        for (int bb = 0; bb < NBT; ++bb) {
          if (bb >= B) break;
#pragma unroll
          for (int j = 0; j < IT; ++j) {
            float x8[8];
            if (XREG) {
#pragma unroll
              for (int q = 0; q < 8; ++q) x8[q] = xr[XREG ? bb : 0][XREG ? j : 0][q];
            } else {
              const float4 a0 = *reinterpret_cast<const float4*>(xs + bb * K + kb + 256 * j);
              const float4 a1 = *reinterpret_cast<const float4*>(xs + bb * K + kb + 256 * j + 4);
              x8[0] = a0.x; x8[1] = a0.y; x8[2] = a0.z; x8[3] = a0.w;
              x8[4] = a1.x; x8[5] = a1.y; x8[6] = a1.z; x8[7] = a1.w;
            }
            float acc = w[j][0] * x8[0];
#pragma unroll
            for (int q = 1; q < 8; ++q) acc = fmaf(w[j][q], x8[q], acc);
            part[bb][j] = acc;
          }
        }
      }
      // Sum over the warp; lane b keeps the total of batch row b.
      float mine = 0.f;
#pragma unroll
      for (int bb = 0; bb < NBT; ++bb) {
        if (bb >= B) break;
        float t = 0.f;
#pragma unroll
        for (int j = 0; j < IT; ++j) t += part[bb][j];
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
        if (lane == bb) mine = t;
      }
      const int slot = stage;
      if (valid) {
        const int need = cs.segs * (pair ? 2 : 1);
        bool finish = need == 1;
        float y = mine, u = 0.f;
        if (!finish) {
          float* cb = comb + ((slot * kConsumerWarps + mrow) * 2) * kMaxB;
          if (lane < B) atomicAdd(cb + (pair && ri >= cs.rows ? kMaxB : 0) + lane, mine);
          __syncwarp();
          __threadfence_block();
          int last = 0;
          if (lane == 0) last = atomicAdd(ccnt + slot * kConsumerWarps + mrow, 1) == need - 1;
          finish = __shfl_sync(0xffffffffu, last, 0) != 0;
          if (finish) {
            __threadfence_block();
            if (lane < B) {
              y = cb[lane];
              u = cb[kMaxB + lane];
              cb[lane] = 0.f;
              cb[kMaxB + lane] = 0.f;
            }
            if (lane == 0) ccnt[slot * kConsumerWarps + mrow] = 0;
          }
        }
        if (finish && lane < B) epilogue(ph, layer, n + mrow, lane, y, u);
      }
      stage_release();
      advance();
      n = e;
    }
  }

  // Output of row n for batch row b (y = the dot product; u = the up row's
  // for a gate/up pair).
  __device__ __forceinline__ void epilogue(int ph, int layer, int n, int b, float y, float u) {
    switch (ph) {
      case kQKV:
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
          const uint32_t uu = __float_as_uint(y);
          const uint32_t ord = (uu & 0x80000000u) ? ~uu : (uu | 0x80000000u);
          const unsigned long long key =
              ((unsigned long long)ord << 32) | (0xffffffffu - (uint32_t)n);
          if (key > wbest) wbest = key;
        }
        break;
      }
    }
  }

  // ---- attention ---------------------------------------------------------
  // Scratch (floats): q [rep][d] | knew [d] | vnew [d] | merge m,l [8][rep][2] | acc [8][rep][d]
  __device__ float* q_s() { return at + 16; }
  __device__ float* k_s() { return q_s() + (p.nq / p.nkv) * p.d; }
  __device__ float* v_s() { return k_s() + p.d; }
  __device__ float* ml_s() { return v_s() + p.d; }
  __device__ float* acc_s() { return ml_s() + kConsumerWarps * (p.nq / p.nkv) * 2; }

  // RMSNorm over one head in a warp + rotate-half RoPE at pos, in place.
  __device__ __forceinline__ void head_norm_rope(float* x, const __nv_bfloat16* gain, int pos) {
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
    const float2* cs = p.rope + (size_t)pos * half;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      if (e >= E) break;
      const int i = lane * E + e;
      const float a = lo[e] * inv * __bfloat162float(gain[i]);
      const float c = hi[e] * inv * __bfloat162float(gain[half + i]);
      const float2 t = cs[i];
      x[i] = a * t.x - c * t.y;
      x[half + i] = c * t.x + a * t.y;
    }
  }

  __device__ __forceinline__ void attn_begin(int layer, int, const Item& x) {
    // The QKV chunks before this end on no barrier: decide quit CTA-wide first.
    quit = consumer_sync_or(quit);
    if (quit) return;
    const int d = p.d, rep = p.nq / p.nkv, qd = p.nq * d, kvd = p.nkv * d;
    const unsigned long long* row = p.xq + (size_t)x.b * (qd + 2 * kvd);
    const uint32_t t1 = tag(layer, 1);
    wait_words(row + x.g * rep * d, rep * d, t1, q_s());
    if (x.owner) {
      wait_words(row + qd + x.g * d, d, t1, k_s());
      wait_words(row + qd + kvd + x.g * d, d, t1, v_s());
    }
    quit = consumer_sync_or(quit);
    if (quit) return;
    tr(layer, 2);
    const LayerDev& Lw = p.layers[layer];
    const int pos = p.pos[x.b];
    if (warp < rep) head_norm_rope(q_s() + warp * d, Lw.q_norm, pos);
    if (x.owner && warp == rep) {
      head_norm_rope(k_s(), Lw.k_norm, pos);
      const size_t off = p.kv.offset(layer, p.seq[x.b], pos, x.g);
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
    const int E = d / 32;
    const float scale = 1.f / sqrtf((float)d);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      m[h] = -INFINITY;
      l[h] = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[h][e] = 0.f;
        qreg[h][e] = (h < rep && e < E) ? q_s()[h * d + lane * E + e] * scale : 0.f;
      }
    }
  }

  // Online-softmax update with one key (k, v given per lane: E elements).
  __device__ __forceinline__ void attend(const float (&kk)[4], const float (&vv)[4], int rep) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (h >= rep) break;
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) s = fmaf(qreg[h][e], kk[e], s);
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      const float mn = fmaxf(m[h], s);
      const float c = expf(m[h] - mn), pr = expf(s - mn);
      l[h] = l[h] * c + pr;
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[h][e] = acc[h][e] * c + pr * vv[e];
      m[h] = mn;
    }
  }

  __device__ __forceinline__ void kv(int, const Item&, int, int nk) {
    if (quit) return;  // no barrier in here: a per-thread exit is harmless
    const unsigned char* st = stage_wait();
    const int d = p.d, rep = p.nq / p.nkv, E = d / 32;
    const __nv_bfloat16* K = reinterpret_cast<const __nv_bfloat16*>(st);
    const __nv_bfloat16* Vv = reinterpret_cast<const __nv_bfloat16*>(st + kWeightBytes / 2);
    for (int j = warp; j < nk && !quit; j += kConsumerWarps) {
      float kk[4] = {0.f, 0.f, 0.f, 0.f}, vv[4] = {0.f, 0.f, 0.f, 0.f};
      if (E == 4) {
        const uint2 ku = *reinterpret_cast<const uint2*>(K + j * d + lane * 4);
        const uint2 vu = *reinterpret_cast<const uint2*>(Vv + j * d + lane * 4);
        kk[0] = lo16(ku.x); kk[1] = hi16(ku.x); kk[2] = lo16(ku.y); kk[3] = hi16(ku.y);
        vv[0] = lo16(vu.x); vv[1] = hi16(vu.x); vv[2] = lo16(vu.y); vv[3] = hi16(vu.y);
      } else {
        const uint32_t ku = *reinterpret_cast<const uint32_t*>(K + j * d + lane * 2);
        const uint32_t vu = *reinterpret_cast<const uint32_t*>(Vv + j * d + lane * 2);
        kk[0] = lo16(ku); kk[1] = hi16(ku);
        vv[0] = lo16(vu); vv[1] = hi16(vu);
      }
      attend(kk, vv, rep);
    }
    stage_release();
    advance();
  }

  __device__ __forceinline__ void attn_end(int layer, int, const Item& x) {
    // No early exit before the first barrier: threads may disagree on quit here.
    const int d = p.d, rep = p.nq / p.nkv, E = d / 32;
    if (x.owner && warp == 0 && !quit) {
      float kk[4] = {0.f, 0.f, 0.f, 0.f}, vv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (e < E) {
          kk[e] = k_s()[lane * E + e];
          vv[e] = v_s()[lane * E + e];
        }
      }
      attend(kk, vv, rep);
    }
    float* ml = ml_s();
    float* ac = acc_s();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (h >= rep) break;
      if (lane == 0) {
        ml[(warp * rep + h) * 2] = m[h];
        ml[(warp * rep + h) * 2 + 1] = l[h];
      }
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (e < E) ac[(warp * rep + h) * d + lane * E + e] = acc[h][e];
    }
    quit = consumer_sync_or(quit);
    if (quit) return;
    const int ns = p.n_splits;
    const uint32_t t2 = tag(layer, 2);
    // merge the warps: thread per (head, dim)
    for (int t = tid; t < rep * d; t += kConsumers) {
      const int h = t / d, c = t % d;
      float M = -INFINITY;
      for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, ml[(w * rep + h) * 2]);
      float L = 0.f, O = 0.f;
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float mw = ml[(w * rep + h) * 2];
        const float f = (mw == -INFINITY) ? 0.f : expf(mw - M);
        L += ml[(w * rep + h) * 2 + 1] * f;
        O += ac[(w * rep + h) * d + c] * f;
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
    if (lane < p.B && wbest) atomicMax(best + lane, wbest);
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
__global__ void __launch_bounds__(kThreads, 1) decode_mega_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  Ring ring;
  ring.stages = smem;
  ring.n = p.n_stages;
  ring.full = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  ring.empty = ring.full + kMaxStages;
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.n_stages; ++s) {
      mbar_init(&ring.full[s], 1);
      mbar_init(&ring.empty[s], kConsumerWarps);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    unsigned long long* best = reinterpret_cast<unsigned long long*>(smem + p.off_misc);
    for (int b = 0; b < kMaxB; ++b) best[b] = 0ull;
  }
  {
    float* cz = reinterpret_cast<float*>(smem + p.off_red);
    const int n = kMaxStages * kConsumerWarps * (2 * kMaxB + 1);
    for (int k = threadIdx.x; k < n; k += blockDim.x) cz[k] = 0.f;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  if (warp == kConsumerWarps) {
    // producer warp: one lane issues, the others go straight to the end
    if ((threadIdx.x & 31) == 0) {
      Producer pr(p, ring);
      walk(p, blockIdx.x, gridDim.x, pr);
      if (p.trace) p.trace[((size_t)blockIdx.x * (p.L + 1) + p.L) * 8 + 3] = now_ns();
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
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace

bool mega_shape_ok(const fs_model* m) {
  const Shape& s = m->s;
  const int rep = s.nq / s.nkv;
  if (rep > 2 || (s.d != 64 && s.d != 128)) return false;
  if (s.V >= 0x7fffffff) return false;
  const int Ks[4] = {s.H, s.q_dim(), s.H, s.I};
  const bool pair[4] = {false, false, true, false};
  for (int i = 0; i < 4; ++i) {
    const mega::ChunkShape cs = mega::chunk_shape(Ks[i], m->q8, pair[i]);
    if ((Ks[i] / cs.segs) % 256 || Ks[i] % cs.segs) return false;
  }
  const mega::ChunkShape lm = mega::chunk_shape(s.H, false, false);
  if ((s.H / lm.segs) % 256) return false;
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
  m->extras = st;
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
    m->extras = nullptr;
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
  MegaState* st = static_cast<MegaState*>(m->extras);
  if (!st) return;
  mega_free(st);
  delete st;
  m->extras = nullptr;
}

// Resets the exchange state after a step was aborted (device error seen).
void mega_reset(fs_model* m) {
  MegaState* st = static_cast<MegaState*>(m->extras);
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
// covered (the caller then uses the general path).
fs_status decode_mega(fs_model* m, const fs_kv* kv, const RowMap& map, int B, const int32_t* tok,
                      const float* h_in, float* h_out, int l0, int l1, bool run_head,
                      float* logits, int32_t* argmax, cudaStream_t stream) {
  MegaState* st = static_cast<MegaState*>(m->extras);
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
  // ~64 keys per attention item, at most one item per CTA
  int ns = (cmax + 63) / 64;
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
  const size_t attn = align_up((16 + rep * s.d + 2 * s.d + mega::kConsumerWarps * rep * 2 +
                                mega::kConsumerWarps * rep * s.d) * 4, 128);
  const size_t redb =
      align_up((size_t)mega::kMaxStages * mega::kConsumerWarps * (2 * mega::kMaxB + 1) * 4, 128);
  const size_t bars = 2 * mega::kMaxStages * 8;
  const size_t misc = 128;
  const size_t fixed = fixed_hs + fixed_xs + attn + redb + bars + misc;
  const size_t budget = 232448;
  int n_stages = (int)((budget - fixed) / mega::kStageBytes);
  n_stages = std::min(n_stages, mega::kMaxStages);
  if (n_stages < 3) return FS_ERR_UNSUPPORTED;
  off = (size_t)n_stages * mega::kStageBytes;
  p.off_hs = (int)off; off += fixed_hs;
  p.off_xs = (int)off; off += fixed_xs;
  p.off_attn = (int)off; off += attn;
  p.off_red = (int)off; off += redb;
  p.off_bar = (int)off; off += bars;
  p.off_misc = (int)off; off += misc;
  p.n_stages = n_stages;
  void* args[] = {&p};
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
