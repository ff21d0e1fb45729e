// Persistent decode forward for batches of 1..4 sequences: one cooperative
// launch (one CTA per SM) runs every block, the final norm, the tied LM head
// and the greedy argmax of one decode step.
//
// Work split of a block (G CTAs, CTA c):
//   A  RMSNorm + QKV projection, row split: CTA c owns rows [a_c, b_c) of
//      Wq|Wk|Wv. Outputs go out as tagged 64-bit words (fp32 value | tag).
//   B  attention fused with the output projection, split by (kv head g,
//      8-wide slice j of the head dimension): the unit normalises and rotates
//      the group's q heads and k (the j = 0 unit appends k, v to the cache),
//      runs the causal softmax over every key of the group, keeps the output
//      o[h][8j .. 8j+8) of each of the group's query heads exactly (no split
//      merge) and multiplies it by the matching 8 rows of Wo^T (a transposed
//      copy made at model creation), adding its share of the O projection to
//      the residual.
//   C  RMSNorm + gate/up + SwiGLU + down, split by intermediate columns: CTA c
//      owns columns [a_c, b_c) of Wg, Wu and the matching rows of Wd^T, so its
//      SwiGLU outputs feed its own share of the down projection, added to the
//      residual.
// Hand-offs between CTAs are 64-bit words (fp32 value | 32-bit tag) written
// with plain stores; a reader polls the words it needs until their tag is the
// current one (tags grow across steps, so nothing is ever cleared and no flag
// or fence is needed). A -> B passes the Q/K/V rows. The residual sums after
// B and after C are reduced without atomics: every contributor (attention
// unit, or CTA of the MLP phase) stores its partial vector in a slot of its
// own; every CTA then sums a slice of about H / G elements over all slots in
// a fixed order (adding the residual the block started the half from) and
// publishes it; every CTA polls the published vector. The sums are therefore
// reproducible bit for bit.
//
// Weight stream. A producer warp (one lane) copies the CTA's weights, the
// group's K/V pages and, for the LM head, its rows of the embedding into a
// ring of shared-memory stages with cp.async.bulk, in the order the consumers
// use them; it runs ahead across phase and block boundaries, since weights do
// not depend on activations. Every consumer warp waits on every chunk and
// arrives on its release barrier (arrival count = consumer warps), so no warp
// can get a full ring ahead of another and a parity wait always refers to the
// chunk it means.
//
// Every wait is bounded by %globaltimer (limit set per launch); on timeout
// the CTA records kErrTimeout, raises the abort flag that every wait checks,
// drains its own bulk copies and returns.
#include <algorithm>

#include "runtime.h"

namespace fs {
namespace fused {

constexpr int kConsumerWarps = 11;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;  // + producer warp
constexpr int kMaxB = 4;
constexpr int kData = 16384;   // main area of a Q8_0 stage
constexpr int kExtra = 2048;   // Q8_0 scale area after it
constexpr int kStageQ8 = kData + kExtra;
constexpr int kStageBf16 = 8 * 2 * 1024;  // eight bf16 rows of K = 1024
constexpr int kMaxStages = 16;
constexpr int kSlice = 8;      // head-dimension slice of one attention unit
constexpr int kMaxRep = 2;     // query heads per kv head
constexpr int kTraceSlots = 16;

enum { kQ8 = 1 };

struct TLayer {
  const void* wo_t;    // Wo^T [nq*d][H] (bf16, or int8 codes)
  const __half* so_t;  // Q8_0: scales of Wo^T rows, [nq*d/32][H]
  const void* wd_t;    // Wd^T [I][H]
  const __half* sd_t;  // Q8_0: [I/32][H]
};

struct Params {
  int L, H, nq, nkv, d, I, V;
  float eps;
  int q8;
  const LayerDev* layers;
  const TLayer* tl;
  const __nv_bfloat16* embed;
  const __nv_bfloat16* final_norm;
  const float2* rope;
  KVView kv;
  int B;
  int seq[kMaxB];
  int pos[kMaxB];
  const int32_t* tokens;
  unsigned long long* xq;    // [B][(nq+2nkv)d] tagged words
  unsigned long long* part_b;  // [n_units][B][H] partial O projections (tagged)
  unsigned long long* part_c;  // [G][B][H] partial down projections (tagged)
  unsigned long long* rsum;    // [2][B][H] reduced residual after attention / after the block
  int n_units;                 // attention units nkv * d/8
  int c_ctas;                // CTAs with intermediate columns
  uint32_t tag0;
  int l0, l1;
  const float* h_in;
  float* h_out;
  int run_head;
  float* logits;
  int32_t* argmax;
  unsigned long long* am_key;
  unsigned int* am_cnt;
  float* capture;
  int capture_stride;
  int* err;
  int* abort_flag;
  unsigned long long wait_ns;
  int withhold_layer;  // debug: phase-A outputs of this layer are never published
  unsigned long long* trace;
  int n_stages;
  int off_r, off_z, off_misc, off_attn, off_tab, off_bar, off_red;
  int bt_in_smem;
  int off_par;  // a copy of these parameters in shared memory (see the kernel)
  int stage_bytes;
  int off_zt;     // [2 slots][2B rows: hi, lo of each batch row][H + 8] bf16 GEMV operands
  int lm_owners;  // warps that consume LM-head chunks (chunk i: warp i % lm_owners)
  int lm_rows;    // rows per LM-head chunk
};

// ---------------------------------------------------------------------------
// Small helpers

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
__device__ __forceinline__ unsigned long long ld_word(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_tag(unsigned long long* p, float v, uint32_t tag) {
  const unsigned long long w = ((unsigned long long)tag << 32) | __float_as_uint(v);
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
__device__ __forceinline__ void mbar_arrive_n(uint64_t* bar, uint32_t n) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(su32(bar)), "r"(n) : "memory");
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
// decision to stop (a timeout seen by one thread) is taken by all at once.
__device__ __forceinline__ bool __syncthreads_or_consumers(bool v) {
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
// Whether a wait first stamped at t0 (0: stamp it now) must stop: it ran
// past `limit`, or, once it has lasted 20 us, another CTA raised the abort
// flag. Only waits that already took long read the one shared flag, so the
// many short waits of a step do not all poll the same word.
__device__ __forceinline__ bool wait_expired(unsigned long long& t0, unsigned long long limit,
                                             const int* abort_flag) {
  const unsigned long long t = now_ns();
  if (t0 == 0) {
    t0 = t;
    return false;
  }
  const unsigned long long dt = t - t0;
  return dt > 20000ull && (dt > limit || aborted(abort_flag));
}
__device__ __forceinline__ float lo16(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float hi16(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
// Warp-level tensor-core operations for the skinny products of decode: A
// (16 x 16 bf16, rows of weights or their transpose) from shared memory by
// ldmatrix, B (16 x 8 bf16) the activation as two bf16 terms per batch row,
// fp32 accumulation.
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
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t (&r)[2]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4],
                                         const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
__device__ __forceinline__ uint32_t word_tag(unsigned long long w) { return (uint32_t)(w >> 32); }
__device__ __forceinline__ float word_value(unsigned long long w) {
  return __uint_as_float((uint32_t)w);
}

__host__ __device__ inline void slice(int N, int G, int c, int& a, int& b) {
  a = (int)((long long)N * c / G);
  b = (int)((long long)N * (c + 1) / G);
}

// Layout of weight rows in a stage (the consumers and the producer agree on
// it): rows packed as in memory (bf16 2H bytes apart, Q8_0 codes H bytes
// apart with their scales at kData), so a chunk of consecutive rows is one
// bulk copy. (A bulk copy per row, to pad the rows against bank conflicts of
// the ldmatrix reads, made the producer's copy issue the bottleneck.)
__host__ __device__ inline int row_stride(int H, bool q8) { return q8 ? H : 2 * H; }
__host__ __device__ inline int rows_cap(int H, bool q8) {  // rows of K = H per chunk
  const int r = q8 ? kData / H : kStageBf16 / (2 * H);
  return r < 16 ? r : 16;
}
__host__ __device__ inline int pairs_cap(int H, bool q8) {
  const int r = q8 ? kData / (2 * H) : rows_cap(H, false) / 2;
  return r < 8 ? r : 8;
}
// End of the QKV chunk from row n (never across the wq|wk|wv boundaries).
__host__ __device__ inline int qkv_chunk_end(int n, int b, int cap, int qd, int kvd) {
  int e = n + cap < b ? n + cap : b;
  if (n < qd) e = e < qd ? e : qd;
  else if (n < qd + kvd) e = e < qd + kvd ? e : qd + kvd;
  return e;
}
// End of the Wd^T chunk from row n: Q8_0 chunks stay within one 32-row block
// (one row of transposed scales).
__host__ __device__ inline int down_chunk_end(int n, int b, int cap, bool q8) {
  int e = n + cap < b ? n + cap : b;
  if (q8) {
    const int blk = (n / 32 + 1) * 32;
    e = e < blk ? e : blk;
  }
  return e;
}

struct Ring {
  unsigned char* stages;
  uint64_t* full;
  uint64_t* empty;
  int n;
};

// Shared-memory copies of the per-layer pointers and the batch's block-table rows.
__device__ __forceinline__ const LayerDev& layer_s(const Params& p, int l) {
  extern __shared__ __align__(1024) unsigned char smem_base[];
  return reinterpret_cast<const LayerDev*>(smem_base + p.off_tab)[l];
}
__device__ __forceinline__ const TLayer& tlayer_s(const Params& p, int l) {
  extern __shared__ __align__(1024) unsigned char smem_base[];
  return reinterpret_cast<const TLayer*>(smem_base + p.off_tab + (size_t)p.L * sizeof(LayerDev))[l];
}
__device__ __forceinline__ size_t kv_off(const Params& p, int layer, int b, int pos, int g) {
  extern __shared__ __align__(1024) unsigned char smem_base[];
  int page;
  if (p.bt_in_smem) {
    const int32_t* bt = reinterpret_cast<const int32_t*>(
        smem_base + p.off_tab + (size_t)p.L * (sizeof(LayerDev) + sizeof(TLayer)));
    page = bt[b * p.kv.pages_per_seq + pos / kPage];
  } else {
    page = p.kv.block_table[(size_t)p.seq[b] * p.kv.pages_per_seq + pos / kPage];
  }
  return (size_t)layer * p.kv.layer_elems() +
         (((size_t)page * p.kv.n_kv_heads + g) * kPage + (pos % kPage)) * p.kv.head_dim;
}

// Tag of hand-off k of block l: 0 Q/K/V rows, 1 O-projection partials, 2 the
// residual after attention, 3 down-projection partials, 4 the block output.
__host__ __device__ __forceinline__ uint32_t tag_of(uint32_t tag0, int l, int l0, int k) {
  return tag0 + 5u * (uint32_t)(l - l0) + (uint32_t)k;
}

// ---------------------------------------------------------------------------
// Out-of-line waiting loops, as free functions taking plain values: a member
// function that is not inlined takes the object's address, which moves the
// whole consumer state (ring cursor, flags, ...) to the stack, and with shared
// memory taking most of L1 every access to it then waits on memory.

// Warp-wide wait until bar1 (if not null) shows phase par1 and bar0 phase
// par0, or the wait runs out; true if it ran out.
__device__ __noinline__ bool warp_wait_slow(uint64_t* bar0, uint32_t par0, uint64_t* bar1,
                                            uint32_t par1, bool quit, unsigned long long limit,
                                            const int* abort_flag) {
  unsigned long long t0 = 0;
  int spins = 0;
  const int lane = threadIdx.x & 31;
  while (true) {
    const bool ok = quit || ((bar1 == nullptr || mbar_test(bar1, par1)) && mbar_test(bar0, par0));
    if (__all_sync(0xffffffffu, ok)) return false;
    __nanosleep(32);
    if ((++spins & 15) == 0) {
      int bad = 0;
      if (lane == 0) bad = wait_expired(t0, limit, abort_flag);
      if (__shfl_sync(0xffffffffu, bad, 0)) return true;
    }
  }
}
// Polls one tagged word until its tag is `want`, backing off; *gave_up is set
// when the wait runs out.
__device__ __noinline__ unsigned long long poll_slow(const unsigned long long* w, uint32_t want,
                                                     unsigned long long limit,
                                                     const int* abort_flag, bool* gave_up) {
  unsigned long long x = 0, t0 = 0;
  int spins = 0;
  unsigned int ns = 32;  // many waiting threads must not flood L2 with loads
  do {
    __nanosleep(ns);
    ns = ns < 256 ? 2 * ns : 256;
    x = ld_word(w);
    if ((++spins & 15) == 0 && wait_expired(t0, limit, abort_flag)) {
      *gave_up = true;
      break;
    }
  } while (word_tag(x) != want);
  return x;
}

// ---------------------------------------------------------------------------
// Producer: issues the bulk copies of every chunk, in consumption order.

struct Producer {
  const Params& p;
  Ring r;
  uint64_t policy;
  unsigned int i = 0;   // chunks issued
  int stage = 0;
  uint32_t parity = 1;  // the first pass over the ring finds every stage free
  bool quit = false;

  __device__ Producer(const Params& pp, Ring rr) : p(pp), r(rr) { policy = evict_first_policy(); }

  __device__ unsigned char* acquire(uint32_t bytes) {
    if (quit) return nullptr;
    const int s = stage;
    unsigned long long t0 = 0;
    int spins = 0;
    while (!mbar_test(&r.empty[s], parity)) {
      // a spinning lane takes issue slots from the consumer warps of its
      // scheduler: sleep between tests
      __nanosleep(128);
      if ((++spins & 15) == 0) {
        if (wait_expired(t0, p.wait_ns, p.abort_flag)) {
          if (!aborted(p.abort_flag)) {
            atomicExch(p.abort_flag, 1);
            atomicCAS(p.err, 0, kErrTimeout);
          }
          quit = true;
          return nullptr;
        }
      }
    }
    mbar_expect_tx(&r.full[s], bytes);
    return r.stages + (size_t)s * p.stage_bytes;
  }
  __device__ __forceinline__ uint64_t* bar() { return &r.full[stage]; }
  __device__ __forceinline__ void advance() {
    ++i;
    if (++stage == r.n) {
      stage = 0;
      parity ^= 1u;
    }
  }

  // Rows [n, n + nr) of a [N][K = H] matrix into `st` from row slot `slot`
  // on, one bulk copy.
  __device__ void copy_rows(unsigned char* st, int slot, const void* w, int n, int nr, bool q8) {
    const uint32_t rb = q8 ? p.H : 2 * p.H;
    const unsigned char* src = static_cast<const unsigned char*>(w) + (size_t)n * rb;
    bulk_load(st + slot * rb, src, nr * rb, bar(), policy);
  }
  // Rows [n, e) of a [N][K = H] matrix (bf16, or Q8_0 codes + scales).
  __device__ void rows(const void* w, const __half* s, int n, int e, bool q8) {
    const int H = p.H, nr = e - n;
    const uint32_t rb = q8 ? H : 2 * H;
    const uint32_t sb = q8 ? H / 16 : 0;
    unsigned char* st = acquire(nr * (rb + sb));
    if (!st) return;
    copy_rows(st, 0, w, n, nr, q8);
    if (q8)
      bulk_load(st + kData, reinterpret_cast<const unsigned char*>(s) + (size_t)n * sb, nr * sb,
                bar(), policy);
    advance();
  }

  __device__ void phase_a(int l, int a, int b) {
    const LayerDev& Lw = layer_s(p, l);
    const bool q8 = p.q8;
    const int qd = p.nq * p.d, kvd = p.nkv * p.d, cap = rows_cap(p.H, q8);
    for (int n = a; n < b && !quit;) {
      const int e = qkv_chunk_end(n, b, cap, qd, kvd);
      const int which = n < qd ? kWq : (n < qd + kvd ? kWk : kWv);
      const int base = which == kWq ? 0 : (which == kWk ? qd : qd + kvd);
      rows(Lw.w[which], Lw.s[which], n - base, e - base, q8);
      n = e;
    }
  }

  __device__ void phase_b(int l, int c, int G) {
    const TLayer& T = tlayer_s(p, l);
    const int H = p.H, d = p.d, ds = d / kSlice, rep = p.nq / p.nkv;
    for (int u = c; u < p.n_units && !quit; u += G) {
      const int g = u / ds, j = u % ds;
      for (int b = 0; b < p.B && !quit; ++b) {
        const int old = p.pos[b];
        for (int j0 = 0; j0 < old && !quit; j0 += kPage) {
          const int nk = min(kPage, old - j0);
          const size_t off = kv_off(p, l, b, j0, g);
          unsigned char* st = acquire(nk * d * 2);
          if (!st) return;
          bulk_load(st, p.kv.k + off, nk * d * 2, bar(), policy);
          advance();
          st = acquire(nk * d * 2);
          if (!st) return;
          bulk_load(st, p.kv.v + off, nk * d * 2, bar(), policy);
          advance();
        }
      }
      for (int h = 0; h < rep && !quit; ++h) {
        const int c0 = (g * rep + h) * d + j * kSlice;
        if (p.q8) {
          unsigned char* st = acquire(kSlice * H + 2 * H);
          if (!st) return;
          bulk_load(st, static_cast<const int8_t*>(T.wo_t) + (size_t)c0 * H, kSlice * H, bar(),
                    policy);
          bulk_load(st + kData, T.so_t + (size_t)(c0 / 32) * H, 2 * H, bar(), policy);
        } else {
          unsigned char* st = acquire(kSlice * 2 * H);
          if (!st) return;
          copy_rows(st, 0, T.wo_t, c0, kSlice, false);
        }
        advance();
      }
    }
  }

  __device__ void phase_c(int l, int a, int b) {
    const LayerDev& Lw = layer_s(p, l);
    const TLayer& T = tlayer_s(p, l);
    const bool q8 = p.q8;
    const int H = p.H, pc = pairs_cap(H, q8);
    const uint32_t rb = q8 ? H : 2 * H;
    const uint32_t sb = q8 ? H / 16 : 0;
    for (int n = a; n < b && !quit;) {
      const int e = min(b, n + pc), nr = e - n;
      unsigned char* st = acquire(2 * nr * (rb + sb));
      if (!st) return;
      copy_rows(st, 0, Lw.w[kWg], n, nr, q8);
      copy_rows(st, pc, Lw.w[kWu], n, nr, q8);
      if (q8) {
        bulk_load(st + kData, reinterpret_cast<const unsigned char*>(Lw.s[kWg]) + (size_t)n * sb,
                  nr * sb, bar(), policy);
        bulk_load(st + kData + pc * sb,
                  reinterpret_cast<const unsigned char*>(Lw.s[kWu]) + (size_t)n * sb, nr * sb,
                  bar(), policy);
      }
      advance();
      n = e;
    }
    const int rc = rows_cap(H, q8);
    for (int n = a; n < b && !quit;) {
      const int e = down_chunk_end(n, b, rc, q8), nr = e - n;
      unsigned char* st = acquire(nr * rb + (q8 ? 2 * H : 0));
      if (!st) return;
      copy_rows(st, 0, T.wd_t, n, nr, q8);
      if (q8) bulk_load(st + kData, T.sd_t + (size_t)(n / 32) * H, 2 * H, bar(), policy);
      advance();
      n = e;
    }
  }

  __device__ void tail(int a, int b) {
    if (!p.run_head) return;
    const int cap = p.lm_rows;
    for (int n = a; n < b && !quit;) {
      const int e = min(b, n + cap);
      rows(p.embed, nullptr, n, e, false);
      n = e;
    }
  }
};

// ---------------------------------------------------------------------------
// Consumers

template <int NB, bool Q8W, int IT, int DQ>
struct Consumer {
  const Params& p;
  Ring r;
  float* rs;    // [B][H] raw residual rows of the current phase input
  float* zs;    // [B][H] gain * residual (the GEMV operand before 1/rms)
  float* zs_base;  // two buffers of zs: phase A / LM head, and phase C
  float* misc;  // ss partials [2][64] | act [kMaxB][128] | o [kMaxB][2][8]
  float* attn;  // q [rep][d] | k [d] | v [d] | warp states
  unsigned long long* best;  // [kMaxB] greedy keys of this CTA
  int* flag;
  unsigned long long wbest[kMaxB] = {0ull, 0ull, 0ull, 0ull};
  unsigned int i = 0;
  int stage = 0;
  uint32_t parity = 0;
  bool quit = false;
  int tid, warp, lane, G, cta;

  __device__ Consumer(const Params& pp, Ring rr, unsigned char* sm) : p(pp), r(rr) {
    rs = reinterpret_cast<float*>(sm + p.off_r);
    zs_base = reinterpret_cast<float*>(sm + p.off_z);
    zs = zs_base;
    misc = reinterpret_cast<float*>(sm + p.off_misc);
    attn = reinterpret_cast<float*>(sm + p.off_attn);
    best = reinterpret_cast<unsigned long long*>(sm + p.off_misc + 4096);
    flag = reinterpret_cast<int*>(sm + p.off_misc + 4096 + 8 * kMaxB);
    tid = threadIdx.x;
    warp = tid >> 5;
    lane = tid & 31;
    G = gridDim.x;
    cta = blockIdx.x;
  }
  float* ss_s = nullptr;                                 // [11][kMaxB] of the current slot
  __device__ float* act_s() { return misc + 128; }       // [kMaxB][128]
  __device__ float* o_s() { return misc + 128 + 512; }   // [kMaxB][kMaxRep][kSlice]
  // Shared-memory layout of the rest of `misc` (bytes): ys [48][4] fp32 at
  // 2816, the greedy keys / flag / counts at 4096, 64 zero bytes at 4160, the
  // tensor-core coefficient rows [8][40] bf16 at 4224, the row table [48] at 4864.
  __device__ float* ys() { return misc + 704; }
  __device__ uint32_t zero_addr() const { return su32(reinterpret_cast<const unsigned char*>(misc) + 4160); }
  __device__ __nv_bfloat16* coef() {
    return reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<unsigned char*>(misc) + 4224);
  }
  __device__ uint32_t* rowaddr() {
    return reinterpret_cast<uint32_t*>(reinterpret_cast<unsigned char*>(misc) + 4864);
  }
  __nv_bfloat16* zt = nullptr;  // the current slot of the tensor-core operand rows
  static constexpr int kCoefStride = 40;  // bf16 per coefficient row (80 bytes)
  __device__ int zt_stride() const { return p.H + 8; }  // bf16 per operand row
  // Shared address of the chunk `ahead` places after the oldest unreleased one.
  __device__ uint32_t stage_addr(int ahead) const {
    int s = stage + ahead;
    if (s >= r.n) s -= r.n;
    return su32(r.stages + (size_t)s * p.stage_bytes);
  }

  // Trace stamp k of (this CTA, layer): the SM's cycle counter (converted on
  // the host with the CTA's own globaltimer / clock pairs at start and end).
  __device__ __forceinline__ void tr(int layer, int k) {
    if (p.trace && tid == 0)
      p.trace[((size_t)cta * (p.L + 1) + layer) * kTraceSlots + k] = clock64();
  }
  __device__ __forceinline__ void give_up() {
    if (!aborted(p.abort_flag)) {
      atomicExch(p.abort_flag, 1);
      atomicCAS(p.err, 0, kErrTimeout);
    }
    quit = true;
  }
  // `quit` of any lane of this warp: the guard of warp-collective work
  // (shuffles, ldmatrix, mma), which every lane must execute or skip
  // together; per-thread quit alone may differ between lanes.
  __device__ __forceinline__ bool warp_quit() const { return __any_sync(0xffffffffu, quit); }

  // Wait (whole warp) for the chunk `ahead` places after the oldest one this
  // warp has not released; returns its stage. Every chunk before it has been
  // waited for by this warp, so the stage's full barrier is in this chunk's
  // phase or the one before it.
  __device__ __forceinline__ const unsigned char* chunk_wait(int ahead = 0) {
    int s = stage + ahead;
    uint32_t par = parity;
    if (s >= r.n) {
      s -= r.n;
      par ^= 1u;
    }
    if (!__all_sync(0xffffffffu, quit || mbar_test(&r.full[s], par)) &&
        warp_wait_slow(&r.full[s], par, nullptr, 0u, quit, p.wait_ns, p.abort_flag))
      give_up();
    return r.stages + (size_t)s * p.stage_bytes;
  }
  __device__ void cursor_advance() {
    ++i;
    if (++stage == r.n) {
      stage = 0;
      parity ^= 1u;
    }
  }
  __device__ void chunk_release() {
    __syncwarp();
    // A thread that gave up has skipped its waits: it must not release a
    // chunk it never saw (an arrival beyond a phase's count is undefined).
    if (lane == 0 && !quit) mbar_arrive(&r.empty[stage]);
    cursor_advance();
  }
  // Wait (whole warp) for the next chunk when this warp alone consumes it and
  // skips the chunks of other warps (W owner warps, ring of n >= W stages):
  // first the release of the chunk n places earlier in the same stage, then
  // the chunk itself. With n >= W the release test cannot see an older phase:
  // this warp waited on a chunk W places back, so every chunk 2n places back
  // has been released.
  __device__ __forceinline__ const unsigned char* chunk_wait_owned() {
    const int s = stage;
    if (!__all_sync(0xffffffffu, quit || (mbar_test(&r.empty[s], parity ^ 1u) &&
                                          mbar_test(&r.full[s], parity))) &&
        warp_wait_slow(&r.full[s], parity, &r.empty[s], parity ^ 1u, quit, p.wait_ns,
                       p.abort_flag))
      give_up();
    return r.stages + (size_t)s * p.stage_bytes;
  }


  // ---- residual input of a phase -----------------------------------------

  static constexpr int kEPT = (NB * IT * 256 + kConsumers - 1) / kConsumers;  // elements / thread
  float inv[NB];
  __device__ __forceinline__ float inv_of(int b) const {
    float v = inv[0];
#pragma unroll
    for (int bb = 1; bb < NB; ++bb)
      if (bb == b) v = inv[bb];
    return v;
  }

  // Gains of this thread's elements (k = tid + 352 e of the [B][H] rows),
  // fetched before the wait for the residual so their latency overlaps it.
  __device__ __forceinline__ void load_gains(const __nv_bfloat16* g, float (&gr)[kEPT]) {
#pragma unroll
    for (int e = 0; e < kEPT; ++e) {
      const int k = tid + e * kConsumers;
      gr[e] = k < p.B * p.H ? __bfloat162float(g[k % p.H]) : 0.f;
    }
  }

  // Polls one tagged word until its tag is `want` (bounded wait); x is the
  // value already loaded.
  __device__ __forceinline__ unsigned long long poll_word(const unsigned long long* w,
                                                          unsigned long long x, uint32_t want) {
    if (word_tag(x) == want || quit) return x;
    bool gave_up = false;
    x = poll_slow(w, want, p.wait_ns, p.abort_flag, &gave_up);
    if (gave_up) give_up();
    return x;
  }


  // This CTA's slice of a residual sum: elements [e0, e1) of the flattened
  // [B][H] rows, each = base[e] (rs: the residual the half started from) plus
  // the partials of contributors 0..n_contrib-1 (slot c at src + c*B*H,
  // tagged tag_in), summed in a fixed order; published to dst with tag_out.
  // Ends on a barrier.
  __device__ __forceinline__ void reduce_slice(const unsigned long long* src, int n_contrib, uint32_t tag_in,
                               unsigned long long* dst, uint32_t tag_out) {
    const int n = p.B * p.H;
    int e0, e1;
    slice(n, G, cta, e0, e1);
    const int E = e1 - e0, total = n_contrib * E;
    float* buf = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(rs) - p.off_r + p.off_red);
    // one thread per contributor first waits for the slice's last word, so
    // only a few threads poll while the partials are still coming
    for (int c = tid; c < n_contrib && E > 0; c += kConsumers) {
      const unsigned long long* last = src + (size_t)c * n + e1 - 1;
      poll_word(last, ld_word(last), tag_in);
    }
    consumer_sync();
    for (int f0 = tid; f0 < total; f0 += 4 * kConsumers) {
      unsigned long long w[4];
      const unsigned long long* ptr[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int f = f0 + u * kConsumers;
        ptr[u] = f < total ? src + (size_t)(f / E) * n + e0 + f % E : src;
        w[u] = f < total ? ld_word(ptr[u]) : 0ull;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int f = f0 + u * kConsumers;
        if (f < total) buf[f] = word_value(poll_word(ptr[u], w[u], tag_in));
      }
    }
    consumer_sync();
    // four threads per element: contributors c = q, q+4, ... in order, then
    // the base value and the four partial sums in a fixed order
    float* part4 = buf + (size_t)n_contrib * E;
    if (tid < 4 * E) {
      const int e = tid >> 2, q = tid & 3;
      float sacc = 0.f;
      for (int c = q; c < n_contrib; c += 4) sacc += buf[c * E + e];
      part4[tid] = sacc;
    }
    consumer_sync();
    if (tid < E && !quit) {
      const float* q4 = part4 + 4 * tid;
      st_tag(dst + e0 + tid, rs[e0 + tid] + ((q4[0] + q4[1]) + (q4[2] + q4[3])), tag_out);
    }
    consumer_sync();  // rs is read above before any thread overwrites it
  }

  // The phase input rows into rs (source: kind >= 0 the published residual
  // rsum[kind] with tag `tag`; -1 the embedding rows of the tokens or h_in),
  // zs = gain * rs, and 1/rms of each row into inv. Ends on a barrier.
  // `slot` (0: phase A and the LM head, 1: phase C) picks the buffers of zs and
  // of the partial sums, so a warp that runs ahead into the next phase never
  // writes what a slower warp still reads.
  __device__ __forceinline__ void gather_norm(int kind, uint32_t tag, const float (&gr)[kEPT], int slot) {
    const int H = p.H, n = p.B * H;
    zs = zs_base + (size_t)slot * n;
    zt = reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<unsigned char*>(misc) - p.off_misc +
                                          p.off_zt) +
         (size_t)slot * 2 * p.B * zt_stride();
    ss_s = misc + slot * 64;
    float ss[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) ss[b] = 0.f;
    unsigned long long w[kEPT];
    const unsigned long long* src = kind >= 0 ? p.rsum + (size_t)kind * n : nullptr;
    if (kind >= 0) {
      // one thread per reducing CTA first waits for the last word of its slice
      for (int c = tid; c < G; c += kConsumers) {
        int a, b;
        slice(n, G, c, a, b);
        if (b > a) poll_word(src + b - 1, ld_word(src + b - 1), tag);
      }
      consumer_sync();
#pragma unroll
      for (int e = 0; e < kEPT; ++e) {
        const int k = tid + e * kConsumers;
        w[e] = k < n ? ld_word(src + k) : 0ull;
      }
#pragma unroll
      for (int e = 0; e < kEPT; ++e) {
        const int k = tid + e * kConsumers;
        if (k < n) w[e] = poll_word(src + k, w[e], tag);
      }
    }
#pragma unroll
    for (int e = 0; e < kEPT; ++e) {
      const int k = tid + e * kConsumers;
      if (k >= n) break;
      const int b = k / H;
      float x;
      if (kind >= 0) {
        x = word_value(w[e]);
      } else if (p.h_in) {
        x = p.h_in[k];
      } else {
        int t = p.tokens[b];
        if (t < 0 || t >= p.V) {
          if (k % H == 0) atomicCAS(p.err, 0, kErrToken);
          t = 0;
        }
        x = __bfloat162float(p.embed[(size_t)t * H + k % H]);
      }
      rs[k] = x;
      const float z = x * gr[e];
      if (Q8W) zs[k] = z;
      // the tensor-core operand: z as hi + lo bf16 terms (rows 2b, 2b + 1)
      const __nv_bfloat16 hi = __float2bfloat16_rn(z);
      const __nv_bfloat16 lo = __float2bfloat16_rn(z - __bfloat162float(hi));
      zt[(size_t)(2 * b) * zt_stride() + k % H] = hi;
      zt[(size_t)(2 * b + 1) * zt_stride() + k % H] = lo;
#pragma unroll
      for (int bb = 0; bb < NB; ++bb)
        if (bb == b) ss[bb] += x * x;
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const float t = warp_sum(ss[b]);
      if (lane == 0) ss_s[warp * kMaxB + b] = t;
    }
    consumer_sync();
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float t = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < kConsumerWarps; ++w2) t += ss_s[w2 * kMaxB + b];
      inv[b] = rsqrtf(t / (float)H + p.eps);
    }
  }

  // Dot products of one weight row (K = H) with every batch row of zs.
  __device__ __forceinline__ void row_dot(const unsigned char* row, const __half* srow,
                                          float (&acc)[NB]) {
    const int H = p.H;
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[b] = 0.f;
#pragma unroll
    for (int it = 0; it < IT; ++it) {
      const int k = lane * 8 + it * 256;
      float w[8];
      float sc = 1.f;
      if (!Q8W) {
        const uint4 u = *reinterpret_cast<const uint4*>(row + 2 * k);
        w[0] = lo16(u.x); w[1] = hi16(u.x); w[2] = lo16(u.y); w[3] = hi16(u.y);
        w[4] = lo16(u.z); w[5] = hi16(u.z); w[6] = lo16(u.w); w[7] = hi16(u.w);
      } else {
        const uint2 u = *reinterpret_cast<const uint2*>(row + k);
        sc = __half2float(srow[k / 32]);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          w[q] = (float)(int8_t)((u.x >> (8 * q)) & 0xff);
          w[4 + q] = (float)(int8_t)((u.y >> (8 * q)) & 0xff);
        }
      }
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        if (b < p.B) {
          const float4 z0 = *reinterpret_cast<const float4*>(zs + b * H + k);
          const float4 z1 = *reinterpret_cast<const float4*>(zs + b * H + k + 4);
          float t = 0.f;
          t = fmaf(w[0], z0.x, t); t = fmaf(w[1], z0.y, t); t = fmaf(w[2], z0.z, t);
          t = fmaf(w[3], z0.w, t); t = fmaf(w[4], z1.x, t); t = fmaf(w[5], z1.y, t);
          t = fmaf(w[6], z1.z, t); t = fmaf(w[7], z1.w, t);
          acc[b] = Q8W ? fmaf(sc, t, acc[b]) : acc[b] + t;
        }
      }
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[b] = warp_sum(acc[b]);
  }

  // ---- tensor-core products ----------------------------------------------

  // ys[r * 4 + b] = sum_k W[r][k] z_b[k] for the R rows whose bf16 data start
  // at the shared addresses rowaddr()[0..R) (K = H): A = the rows (16-row
  // tiles), B = the 2B operand rows of zt (hi and lo term of each batch row),
  // so column 2b + t of the product is term t of batch row b. Work items are
  // (row tile, block of 8 k-steps), warp w taking items w, w + 11, ...; the
  // items' partial sums meet in shared memory and are added in a fixed order.
  // Ends on a barrier.
  __device__ __forceinline__ void mma_rows(int R) {
    const uint32_t* ra = rowaddr();
    float* part = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(rs) - p.off_r + p.off_red);
    const int nkb = p.H / 128, mt = (R + 15) / 16, items = mt * nkb, twoB = 2 * p.B;
    const uint32_t z0 = su32(zt), zrow = (uint32_t)zt_stride() * 2, zero = zero_addr();
    for (int it = warp; it < items; it += kConsumerWarps) {
      const int m = it / nkb, kb0 = (it % nkb) * 8;
      const int row = m * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
      const bool arow = row < R;
      uint32_t aaddr = arow ? ra[row] + ((lane >> 4) << 4) + kb0 * 32 : zero;
      const int n = lane & 7;
      const bool brow = n < twoB;
      uint32_t baddr = brow ? z0 + n * zrow + (((lane >> 3) & 1) << 4) + kb0 * 32 : zero;
      const uint32_t astep = arow ? 32u : 0u, bstep = brow ? 32u : 0u;
      float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 8; ks += 2) {
        uint32_t a[4], b[2], a2[4], b2[2];
        ldsm_x4(aaddr, a);
        ldsm_x2(baddr, b);
        ldsm_x4(aaddr + astep, a2);
        ldsm_x2(baddr + bstep, b2);
        mma16816(d0, a, b);
        mma16816(d1, a2, b2);
        aaddr += 2 * astep;
        baddr += 2 * bstep;
      }
      const int g = lane >> 2, q = lane & 3;
      part[(it * 16 + g) * 4 + q] = (d0[0] + d1[0]) + (d0[1] + d1[1]);
      part[(it * 16 + g + 8) * 4 + q] = (d0[2] + d1[2]) + (d0[3] + d1[3]);
    }
    consumer_sync();
    float* y = ys();
    for (int t = tid; t < R * 4; t += kConsumers) {
      const int rr = (t >> 2) & 15, q = t & 3, m = t >> 6;
      float sum = 0.f;
      for (int kb = 0; kb < nkb; ++kb) sum += part[((m * nkb + kb) * 16 + rr) * 4 + q];
      y[t] = sum;
    }
    consumer_sync();
  }

  // The coefficient rows of mma_cols from fp32 values v(b, r), r < KR (zero
  // from KR to 32): row 2b holds the bf16 hi term, row 2b + 1 the lo term.
  template <class V>
  __device__ __forceinline__ void fill_coef(int KR, V&& v) {
    __nv_bfloat16* c = coef();
    for (int t = tid; t < 8 * 32; t += kConsumers) {
      const int row = t >> 5, r = t & 31, b = row >> 1;
      float x = 0.f;
      if (b < p.B && r < KR) x = v(b, r);
      const __nv_bfloat16 hi = __float2bfloat16_rn(x);
      c[row * kCoefStride + r] = (row & 1) ? __float2bfloat16_rn(x - __bfloat162float(hi)) : hi;
    }
  }

  // For every column c < H of a transposed matrix held as KR rows (row r's
  // bf16 data at rowaddr()[r], KR <= 32) and the coefficients of coef():
  // out(c, b) = sum_r W[r][c] coef_b[r], on the tensor cores with A = W^T
  // (ldmatrix .trans), one 16-column tile per item, warp w taking tiles
  // w, w + 11, ...; emit(c, b, value) for each column and batch row.
  template <class F>
  __device__ __forceinline__ void mma_cols(int KR, F&& emit) {
    const uint32_t* ra = rowaddr();
    const int ksn = (KR + 15) / 16, tiles = p.H / 16, twoB = 2 * p.B;
    const uint32_t c0 = su32(coef()), zero = zero_addr();
    const int g = lane >> 2, q = lane & 3, n = lane & 7;
    for (int t = warp; t < tiles; t += kConsumerWarps) {
      float d[4] = {0.f, 0.f, 0.f, 0.f};
      for (int ks = 0; ks < ksn; ++ks) {
        const int r = ks * 16 + (lane & 7) + (lane >> 4) * 8;
        const int col = t * 16 + ((lane >> 3) & 1) * 8;
        const uint32_t aaddr = r < KR ? ra[r] + col * 2 : zero;
        const uint32_t baddr =
            n < twoB ? c0 + n * (kCoefStride * 2) + ks * 32 + (((lane >> 3) & 1) << 4) : zero;
        uint32_t a[4], b[2];
        ldsm_x4_t(aaddr, a);
        ldsm_x2(baddr, b);
        mma16816(d, a, b);
      }
      if (q < p.B) {
        emit(t * 16 + g, q, d[0] + d[1]);
        emit(t * 16 + g + 8, q, d[2] + d[3]);
      }
    }
  }

  // One LM-head chunk (nr <= 8 rows of the embedding at the padded stride) on
  // this warp: logits of every batch row, folded into the greedy keys.
  __device__ __forceinline__ void lm_rows_mma(const unsigned char* st, int n0, int nr) {
    const uint32_t rs2 = (uint32_t)row_stride(p.H, false), zero = zero_addr();
    const int row = (lane & 7) + ((lane >> 3) & 1) * 8;
    const bool arow = row < nr;
    uint32_t aaddr = arow ? su32(st) + row * rs2 + ((lane >> 4) << 4) : zero;
    const int n = lane & 7;
    const bool brow = n < 2 * p.B;
    uint32_t baddr = brow ? su32(zt) + n * zt_stride() * 2 + (((lane >> 3) & 1) << 4) : zero;
    const uint32_t astep = arow ? 32u : 0u, bstep = brow ? 32u : 0u;
    float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
    for (int ks = 0; ks < p.H / 16; ks += 2) {
      uint32_t a[4], b[2], a2[4], b2[2];
      ldsm_x4(aaddr, a);
      ldsm_x2(baddr, b);
      ldsm_x4(aaddr + astep, a2);
      ldsm_x2(baddr + bstep, b2);
      mma16816(d0, a, b);
      mma16816(d1, a2, b2);
      aaddr += 2 * astep;
      baddr += 2 * bstep;
    }
    const int g = lane >> 2, q = lane & 3;
    if (g < nr && q < p.B) fold_logit(q, n0 + g, ((d0[0] + d1[0]) + (d0[1] + d1[1])) * inv_of(q));
  }

  // ---- phase A: RMSNorm + QKV rows --------------------------------------

  __device__ __forceinline__ void capture_rows(int slot) {
    if (!p.capture || cta != 0) return;
    for (int k = tid; k < p.B * p.H; k += kConsumers) {
      const int b = k / p.H, e = k % p.H;
      p.capture[((size_t)slot * p.capture_stride + b) * p.H + e] = rs[k];
    }
  }

  __device__ __forceinline__ void phase_a(int l, int a, int b) {
    tr(l, 0);
    const LayerDev& Lw = layer_s(p, l);
    float gr[kEPT];
    load_gains(Lw.attn_norm, gr);
    if (l == p.l0) {
      gather_norm(-1, 0u, gr, 0);
    } else {
      reduce_slice(p.part_c, p.c_ctas, tag_of(p.tag0, l - 1, p.l0, 3), p.rsum + (size_t)p.B * p.H,
                   tag_of(p.tag0, l - 1, p.l0, 4));
      tr(l, 11);
      gather_norm(1, tag_of(p.tag0, l - 1, p.l0, 4), gr, 0);
    }
    tr(l, 1);
    capture_rows(l);
    const int qkvd = (p.nq + 2 * p.nkv) * p.d;
    const int qd = p.nq * p.d, kvd = p.nkv * p.d, cap = rows_cap(p.H, Q8W);
    const uint32_t tag = tag_of(p.tag0, l, p.l0, 0);
    const bool publish = l != p.withhold_layer;
    if constexpr (!Q8W) {
      // every chunk of the phase resident at once, then the tensor cores
      int nch = 0;
      for (int n = a; n < b; n = qkv_chunk_end(n, b, cap, qd, kvd)) ++nch;
      for (int c = 0; c < nch; ++c) chunk_wait(c);
      if (warp == 0) {
        const int rs2 = row_stride(p.H, false);
        int c = 0;
        for (int n = a; n < b; ++c) {
          const int e = qkv_chunk_end(n, b, cap, qd, kvd);
          for (int i = lane; i < e - n; i += 32) rowaddr()[n - a + i] = stage_addr(c) + i * rs2;
          n = e;
        }
      }
      consumer_sync();
      mma_rows(b - a);
      for (int t = tid; t < (b - a) * p.B; t += kConsumers) {
        const int rr = t / p.B, bb = t % p.B;
        if (publish && !quit)
          st_tag(p.xq + (size_t)bb * qkvd + a + rr, ys()[rr * 4 + bb] * inv_of(bb), tag);
      }
      for (int c = 0; c < nch; ++c) chunk_release();
      tr(l, 2);
      return;
    }
    const int rb = Q8W ? p.H : 2 * p.H;
    for (int n = a; n < b;) {
      const int e = qkv_chunk_end(n, b, cap, qd, kvd), nr = e - n;
      const unsigned char* st = chunk_wait();
      int r0 = (warp - (n - a)) % kConsumerWarps;
      if (r0 < 0) r0 += kConsumerWarps;
      if (!warp_quit()) {
        for (int rr = r0; rr < nr; rr += kConsumerWarps) {
          float acc[NB];
          row_dot(st + rr * rb,
                  reinterpret_cast<const __half*>(st + kData) + rr * (p.H / 32), acc);
          if (lane == 0 && publish) {
#pragma unroll
            for (int bb = 0; bb < NB; ++bb)
              if (bb < p.B) st_tag(p.xq + (size_t)bb * qkvd + n + rr, acc[bb] * inv[bb], tag);
          }
        }
      }
      chunk_release();
      n = e;
    }
    tr(l, 2);
  }

  // ---- phase B: attention units with their share of the O projection ------

  // Per-lane constants of one head's RMSNorm + RoPE (elements lane*E + e of
  // both halves, E = d/64).
  struct HeadConst {
    float g_lo[2], g_hi[2];
    float2 cs[2];
  };
  __device__ __forceinline__ void head_const(const __nv_bfloat16* gain, int pos, HeadConst& hc) {
    const int half = p.d / 2, E = p.d / 64;
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
  // Poll one head's d tagged words of xq into x_lo/x_hi (elements lane*E+e).
  __device__ __forceinline__ void poll_head(const unsigned long long* src, uint32_t want,
                                            float (&lo)[2], float (&hi)[2]) {
    const int half = p.d / 2, E = p.d / 64;
    unsigned long long xs[2][2];
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
      for (int part = 0; part < 2; ++part)
        xs[e][part] = e < E ? ld_word(src + lane * E + e + part * half) : 0ull;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      lo[e] = hi[e] = 0.f;
      if (e >= E) continue;
      const int i = lane * E + e;
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        const unsigned long long x = poll_word(src + i + part * half, xs[e][part], want);
        (part ? hi[e] : lo[e]) = word_value(x);
      }
    }
  }
  // RMSNorm over the head (warp) + rotate-half RoPE; writes the d values.
  __device__ __forceinline__ void head_norm_rope(float (&lo)[2], float (&hi)[2],
                                                 const HeadConst& hc, float scale, float* out) {
    const int half = p.d / 2, E = p.d / 64;
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 2; ++e)
      if (e < E) ss += lo[e] * lo[e] + hi[e] * hi[e];
    ss = warp_sum(ss);
    const float inv = rsqrtf(ss / (float)p.d + p.eps);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      if (e >= E) break;
      const int i = lane * E + e;
      const float a = lo[e] * inv * hc.g_lo[e];
      const float c = hi[e] * inv * hc.g_hi[e];
      out[i] = (a * hc.cs[e].x - c * hc.cs[e].y) * scale;
      out[half + i] = (c * hc.cs[e].x + a * hc.cs[e].y) * scale;
    }
  }

  __device__ float* q_sm() { return attn; }                         // [rep][d]
  __device__ float* k_sm() { return attn + kMaxRep * 128; }         // [d]
  __device__ float* v_sm() { return attn + kMaxRep * 128 + 128; }   // [d]
  __device__ float* st_sm() { return attn + kMaxRep * 128 + 256; }  // [11][rep][2 + 8]

  // q heads, k and v of (row b, group g) into shared memory; the j = 0 unit
  // also appends k and v (bf16) to the cache. Ends on a barrier.
  __device__ __forceinline__ void attn_prep(int l, int b, int g, int j) {
    const int d = p.d, rep = p.nq / p.nkv, qd = p.nq * d, kvd = p.nkv * d;
    const int qkvd = qd + 2 * kvd, pos = p.pos[b];
    const LayerDev& Lw = layer_s(p, l);
    const unsigned long long* row = p.xq + (size_t)b * qkvd;
    const uint32_t want = tag_of(p.tag0, l, p.l0, 0);
    if (warp < rep) {
      HeadConst hc;
      head_const(Lw.q_norm, pos, hc);
      float lo[2], hi[2];
      poll_head(row + (g * rep + warp) * d, want, lo, hi);
      head_norm_rope(lo, hi, hc, rsqrtf((float)d), q_sm() + warp * d);
    } else if (warp == rep) {
      HeadConst hc;
      head_const(Lw.k_norm, pos, hc);
      float lo[2], hi[2];
      poll_head(row + qd + g * d, want, lo, hi);
      head_norm_rope(lo, hi, hc, 1.f, k_sm());
      __syncwarp();
      const size_t off = kv_off(p, l, b, pos, g);
      for (int i2 = lane; i2 < d; i2 += 32) {
        const __nv_bfloat16 kb = __float2bfloat16_rn(k_sm()[i2]);
        if (j == 0 && !quit) p.kv.k[off + i2] = kb;
        k_sm()[i2] = __bfloat162float(kb);
      }
    } else if (warp == rep + 1) {
      float lo[2], hi[2];
      poll_head(row + qd + kvd + g * d, want, lo, hi);
      const int half = d / 2, E = d / 64;
      const size_t off = kv_off(p, l, b, pos, g);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        if (e >= E) break;
        const int i2 = lane * E + e;
        const __nv_bfloat16 vl = __float2bfloat16_rn(lo[e]);
        const __nv_bfloat16 vh = __float2bfloat16_rn(hi[e]);
        if (j == 0 && !quit) {
          p.kv.v[off + i2] = vl;
          p.kv.v[off + half + i2] = vh;
        }
        v_sm()[i2] = __bfloat162float(vl);
        v_sm()[half + i2] = __bfloat162float(vh);
      }
    }
    consumer_sync();
  }

  // Online-softmax state of this lane: lane = (key kk = lane >> 2, quarter
  // qq = lane & 3); the quarter holds dims [qq*d/4, (qq+1)*d/4) of the score
  // dot products and dims 8j + 2qq, 8j + 2qq + 1 of the output slice.
  struct AttnState {
    float m[kMaxRep], l[kMaxRep], o[kMaxRep][2];
  };

  // One group of 8 keys (kk valid iff kk < nk): scores, update, P*V.
  // q holds the lane's quarter of each head in rotated 8-element blocks:
  // block c of the registers is block (c + kk) % (DQ/8) of the quarter, so
  // the 8 key lanes of one quarter read different bank groups of their keys.
  __device__ __forceinline__ void attend8(const float (&q)[kMaxRep][DQ], const __nv_bfloat16* Kp,
                                          const __nv_bfloat16* Vp, int nk, int vcol, int rep,
                                          AttnState& S) {
    constexpr int NC = DQ / 8;
    const int kk = lane >> 2, qq = lane & 3, d = 4 * DQ;
    const bool valid = kk < nk;
    float s[kMaxRep];
#pragma unroll
    for (int h = 0; h < kMaxRep; ++h) s[h] = 0.f;
    if (valid) {
      const __nv_bfloat16* krow = Kp + kk * d + qq * DQ;
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        const uint4 u = *reinterpret_cast<const uint4*>(krow + ((c + kk) % NC) * 8);
        const float kf[8] = {lo16(u.x), hi16(u.x), lo16(u.y), hi16(u.y),
                             lo16(u.z), hi16(u.z), lo16(u.w), hi16(u.w)};
#pragma unroll
        for (int h = 0; h < kMaxRep; ++h)
#pragma unroll
          for (int t = 0; t < 8; ++t) s[h] = fmaf(q[h][c * 8 + t], kf[t], s[h]);
      }
    }
    float vv[2] = {0.f, 0.f};
    if (valid) {
      const uint32_t u = *reinterpret_cast<const uint32_t*>(Vp + kk * d + vcol + 2 * qq);
      vv[0] = lo16(u);
      vv[1] = hi16(u);
    }
#pragma unroll
    for (int h = 0; h < kMaxRep; ++h) {
      if (h >= rep) break;
      float t = s[h];
      t += __shfl_xor_sync(0xffffffffu, t, 1);
      t += __shfl_xor_sync(0xffffffffu, t, 2);
      t = valid ? t : -INFINITY;
      float mx = t;
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float mn = fmaxf(S.m[h], mx);
      const float alpha = (S.m[h] == -INFINITY) ? 0.f : expf(S.m[h] - mn);
      const float pr = valid ? expf(t - mn) : 0.f;
      S.m[h] = mn;
      // l: one copy per key lane (summed over keys at the end); quarters
      // other than 0 keep l at zero.
      S.l[h] = S.l[h] * alpha + (qq == 0 ? pr : 0.f);
      S.o[h][0] = fmaf(pr, vv[0], S.o[h][0] * alpha);
      S.o[h][1] = fmaf(pr, vv[1], S.o[h][1] * alpha);
    }
  }

  __device__ __forceinline__ void attn_keys(int l, int b, int g, int j, AttnState& S) {
    const int rep = p.nq / p.nkv, old = p.pos[b];
    float q[kMaxRep][DQ];
    const int qq = lane & 3;
    constexpr int NC = DQ / 8;
    const int kk = lane >> 2;
#pragma unroll
    for (int h = 0; h < kMaxRep; ++h)
#pragma unroll
      for (int c = 0; c < NC; ++c)
#pragma unroll
        for (int t = 0; t < 8; ++t)
          q[h][c * 8 + t] = h < rep ? q_sm()[h * 4 * DQ + qq * DQ + ((c + kk) % NC) * 8 + t] : 0.f;
#pragma unroll
    for (int h = 0; h < kMaxRep; ++h) {
      S.m[h] = -INFINITY;
      S.l[h] = 0.f;
      S.o[h][0] = S.o[h][1] = 0.f;
    }
    const int vcol = j * kSlice;
    // groups of 8 keys: group gi covers keys [8 gi, 8 gi + 8); warp w takes
    // groups w, w + 11, ...; a page holds 8 groups.
    for (int j0 = 0; j0 < old; j0 += kPage) {
      const int nk = min(kPage, old - j0);
      const __nv_bfloat16* Kp = reinterpret_cast<const __nv_bfloat16*>(chunk_wait(0));
      const __nv_bfloat16* Vp = reinterpret_cast<const __nv_bfloat16*>(chunk_wait(1));
      if (!warp_quit()) {
        const int g0 = j0 / 8, g1 = (j0 + nk + 7) / 8;
        int gi = g0 + ((warp - g0) % kConsumerWarps + kConsumerWarps) % kConsumerWarps;
        for (; gi < g1; gi += kConsumerWarps) {
          const int kbase = gi * 8 - j0;
          attend8(q, Kp + (size_t)kbase * 4 * DQ, Vp + (size_t)kbase * 4 * DQ,
                      min(8, nk - kbase), vcol, rep, S);
        }
      }
      chunk_release();  // K
      chunk_release();  // V
    }
    (void)l;
    (void)g;
  }

  // The new key (position pos, from k_sm / v_sm) on warp 0, then the merge of
  // the warps' states into o_s[b][h][t]. Ends on a barrier.
  __device__ __forceinline__ void attn_finish(int b, int j, AttnState& S) {
    const int rep = p.nq / p.nkv, d = 4 * DQ, qq = lane & 3, kk = lane >> 2;
    if (warp == 0 && !warp_quit()) {
      float s[kMaxRep];
#pragma unroll
      for (int h = 0; h < kMaxRep; ++h) {
        float t = 0.f;
        if (kk == 0 && h < rep)
#pragma unroll
          for (int c = 0; c < DQ; ++c) t = fmaf(q_sm()[h * d + qq * DQ + c], k_sm()[qq * DQ + c], t);
        t += __shfl_xor_sync(0xffffffffu, t, 1);
        t += __shfl_xor_sync(0xffffffffu, t, 2);
        s[h] = __shfl_sync(0xffffffffu, t, 0);
      }
#pragma unroll
      for (int h = 0; h < kMaxRep; ++h) {
        if (h >= rep) break;
        const float mn = fmaxf(S.m[h], s[h]);
        const float alpha = (S.m[h] == -INFINITY) ? 0.f : expf(S.m[h] - mn);
        const float pr = (kk == 0) ? expf(s[h] - mn) : 0.f;
        S.m[h] = mn;
        S.l[h] = S.l[h] * alpha + (qq == 0 ? pr : 0.f);
        const float v0 = v_sm()[j * kSlice + 2 * qq], v1 = v_sm()[j * kSlice + 2 * qq + 1];
        S.o[h][0] = fmaf(pr, v0, S.o[h][0] * alpha);
        S.o[h][1] = fmaf(pr, v1, S.o[h][1] * alpha);
      }
    }
    // reduce over the 8 key lanes (same quarter): lanes qq = 0..3 keep the sums
#pragma unroll
    for (int h = 0; h < kMaxRep; ++h) {
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        S.l[h] += __shfl_xor_sync(0xffffffffu, S.l[h], o);
        S.o[h][0] += __shfl_xor_sync(0xffffffffu, S.o[h][0], o);
        S.o[h][1] += __shfl_xor_sync(0xffffffffu, S.o[h][1], o);
      }
    }
    float* ws = st_sm();  // [warp][h][0: m, 1: l, 2..9: o]
    if (lane < 4) {
#pragma unroll
      for (int h = 0; h < kMaxRep; ++h) {
        if (h >= rep) break;
        float* e = ws + (warp * kMaxRep + h) * 10;
        if (lane == 0) {
          e[0] = S.m[h];
          e[1] = S.l[h];
        }
        e[2 + 2 * lane] = S.o[h][0];
        e[3 + 2 * lane] = S.o[h][1];
      }
    }
    consumer_sync();
    if (tid < rep * kSlice) {
      const int h = tid / kSlice, t = tid % kSlice;
      float M = -INFINITY;
      for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, ws[(w * kMaxRep + h) * 10]);
      float Lsum = 0.f, O = 0.f;
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float* e = ws + (w * kMaxRep + h) * 10;
        const float f = (e[0] == -INFINITY) ? 0.f : expf(e[0] - M);
        Lsum += e[1] * f;
        O += e[2 + t] * f;
      }
      o_s()[(b * kMaxRep + h) * kSlice + t] = O / Lsum;
    }
    consumer_sync();
  }

  // Stores one contributor's partial (per batch row: 4 consecutive elements
  // from n4*4) into its slot `slot` ([B][H] words) with tag `tag`.
  __device__ __forceinline__ void contribute(unsigned long long* slot, int n4,
                                             const float (&a)[NB][4], uint32_t tag) {
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (b >= p.B) break;
      unsigned long long* dst = slot + (size_t)b * p.H + 4 * n4;
#pragma unroll
      for (int e = 0; e < 4; ++e) st_tag(dst + e, a[b][e], tag);
    }
  }

  // acc4[b][0..3] += s[b] * W[row][4 n4 .. 4 n4 + 4) for one row of a
  // transposed matrix in shared memory (bf16, or Q8_0 codes with a scale row).
  __device__ __forceinline__ void axpy_row(const unsigned char* row, const __half* srow, int n4,
                                           const float (&s)[NB], float (&acc4)[NB][4]) {
    float w[4];
    if (!Q8W) {
      const uint2 u = *reinterpret_cast<const uint2*>(row + 8 * n4);
      w[0] = lo16(u.x); w[1] = hi16(u.x); w[2] = lo16(u.y); w[3] = hi16(u.y);
    } else {
      const uint32_t u = *reinterpret_cast<const uint32_t*>(row + 4 * n4);
      const uint2 sv = *reinterpret_cast<const uint2*>(srow + 4 * n4);
      const float s0 = __half2float(__ushort_as_half((unsigned short)(sv.x & 0xffff)));
      const float s1 = __half2float(__ushort_as_half((unsigned short)(sv.x >> 16)));
      const float s2 = __half2float(__ushort_as_half((unsigned short)(sv.y & 0xffff)));
      const float s3 = __half2float(__ushort_as_half((unsigned short)(sv.y >> 16)));
      w[0] = (float)(int8_t)(u & 0xff) * s0;
      w[1] = (float)(int8_t)((u >> 8) & 0xff) * s1;
      w[2] = (float)(int8_t)((u >> 16) & 0xff) * s2;
      w[3] = (float)(int8_t)((u >> 24) & 0xff) * s3;
    }
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc4[b][e] = fmaf(s[b], w[e], acc4[b][e]);
  }

  __device__ __forceinline__ void phase_b(int l) {
    tr(l, 3);
    const int d = p.d, ds = d / kSlice, rep = p.nq / p.nkv, H = p.H;
    for (int u = cta; u < p.n_units; u += G) {
      const int g = u / ds, j = u % ds;
      for (int b = 0; b < p.B; ++b) {
        attn_prep(l, b, g, j);
        if (b == 0) tr(l, 4);
        AttnState S;
        attn_keys(l, b, g, j, S);
        if (b == 0) tr(l, 13);
        attn_finish(b, j, S);
      }
      tr(l, 5);
      if constexpr (!Q8W) {
        // O projection share on the tensor cores: the unit's 8 rows of Wo^T
        // per query head (one chunk each) times its o values
        for (int h = 0; h < rep; ++h) chunk_wait(h);
        const int rs2 = row_stride(H, false);
        if (warp == 0 && lane < rep * kSlice)
          rowaddr()[lane] = stage_addr(lane / kSlice) + (lane % kSlice) * rs2;
        fill_coef(rep * kSlice, [&](int bb, int r) {
          return o_s()[(bb * kMaxRep + r / kSlice) * kSlice + r % kSlice];
        });
        consumer_sync();
        unsigned long long* slot = p.part_b + (size_t)u * p.B * H;
        const uint32_t t1 = tag_of(p.tag0, l, p.l0, 1);
        mma_cols(rep * kSlice, [&](int c, int bb, float v) {
          if (!quit) st_tag(slot + (size_t)bb * H + c, v, t1);
        });
        for (int h = 0; h < rep; ++h) chunk_release();
        continue;
      }
      // O projection share: Wo^T rows (g*rep + h)*d + 8j + t
      const int n4 = tid;
      float acc4[NB][4];
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc4[b][e] = 0.f;
      for (int h = 0; h < rep; ++h) {
        const unsigned char* st = chunk_wait();
        if (!quit && n4 < H / 4) {
          const int rb = Q8W ? H : 2 * H;
          const __half* srow = reinterpret_cast<const __half*>(st + kData);
#pragma unroll 4
          for (int t = 0; t < kSlice; ++t) {
            float s[NB];
#pragma unroll
            for (int b = 0; b < NB; ++b) s[b] = o_s()[(b * kMaxRep + h) * kSlice + t];
            axpy_row(st + t * rb, srow, n4, s, acc4);
          }
        }
        chunk_release();
      }
      if (!quit && n4 < H / 4)
        contribute(p.part_b + (size_t)u * p.B * H, n4, acc4, tag_of(p.tag0, l, p.l0, 1));
    }
    tr(l, 6);
  }

  // ---- phase C: RMSNorm + gate/up + SwiGLU + down share ------------------

  __device__ __forceinline__ void phase_c(int l, int a, int b) {
    tr(l, 7);
    const LayerDev& Lw = layer_s(p, l);
    float gr[kEPT];
    load_gains(Lw.ffn_norm, gr);
    reduce_slice(p.part_b, p.n_units, tag_of(p.tag0, l, p.l0, 1), p.rsum,
                 tag_of(p.tag0, l, p.l0, 2));
    tr(l, 12);
    gather_norm(0, tag_of(p.tag0, l, p.l0, 2), gr, 1);
    tr(l, 8);
    const int H = p.H, pc = pairs_cap(H, Q8W);
    if constexpr (!Q8W) {
      // gate/up rows: all chunks resident, one tensor-core pass over 2P rows
      const int P = b - a, rs2 = row_stride(H, false);
      const int ngu = (P + pc - 1) / pc;
      for (int c = 0; c < ngu; ++c) chunk_wait(c);
      if (warp == 0)
        for (int q2 = lane; q2 < P; q2 += 32) {
          const uint32_t st2 = stage_addr(q2 / pc);
          rowaddr()[q2] = st2 + (q2 % pc) * rs2;
          rowaddr()[P + q2] = st2 + (pc + q2 % pc) * rs2;
        }
      consumer_sync();
      mma_rows(2 * P);
      for (int t = tid; t < P * p.B; t += kConsumers) {
        const int q2 = t / p.B, bb = t % p.B;
        const float y = ys()[q2 * 4 + bb] * inv_of(bb), z = ys()[(P + q2) * 4 + bb] * inv_of(bb);
        act_s()[bb * 128 + q2] = y / (1.f + expf(-y)) * z;
      }
      for (int c = 0; c < ngu; ++c) chunk_release();
      tr(l, 9);
      // down share: the CTA's P rows of Wd^T times its SwiGLU outputs
      const int rc = rows_cap(H, false), nd = (P + rc - 1) / rc;
      for (int c = 0; c < nd; ++c) chunk_wait(c);
      consumer_sync();  // act_s complete; rowaddr free again
      if (warp == 0)
        for (int j = lane; j < P; j += 32) rowaddr()[j] = stage_addr(j / rc) + (j % rc) * rs2;
      fill_coef(P, [&](int bb, int r) { return act_s()[bb * 128 + r]; });
      consumer_sync();
      unsigned long long* slot = p.part_c + (size_t)cta * p.B * H;
      const uint32_t t3 = tag_of(p.tag0, l, p.l0, 3);
      mma_cols(P, [&](int c, int bb, float v) {
        if (!quit) st_tag(slot + (size_t)bb * H + c, v, t3);
      });
      for (int c = 0; c < nd; ++c) chunk_release();
      tr(l, 10);
    } else {
      phase_c_q8(l, a, b);
    }
  }

  // Phase C with Q8_0 weights on the CUDA cores (codes widened in registers).
  __device__ void phase_c_q8(int l, int a, int b) {
    const int H = p.H, pc = pairs_cap(H, Q8W), rb = Q8W ? H : 2 * H, sb = Q8W ? H / 32 : 0;
    for (int n = a; n < b;) {
      const int e = min(b, n + pc), nr = e - n;
      const unsigned char* st = chunk_wait();
      int r0 = (warp - (n - a)) % kConsumerWarps;
      if (r0 < 0) r0 += kConsumerWarps;
      if (!warp_quit()) {
        for (int rr = r0; rr < nr; rr += kConsumerWarps) {
          float gv[NB], uv[NB];
          const __half* sg = reinterpret_cast<const __half*>(st + kData) + rr * sb;
          const __half* su = reinterpret_cast<const __half*>(st + kData) + (pc + rr) * sb;
          row_dot(st + rr * rb, sg, gv);
          row_dot(st + (pc + rr) * rb, su, uv);
          if (lane == 0) {
#pragma unroll
            for (int bb = 0; bb < NB; ++bb) {
              if (bb >= p.B) break;
              const float y = gv[bb] * inv[bb], z = uv[bb] * inv[bb];
              act_s()[bb * 128 + (n - a) + rr] = y / (1.f + expf(-y)) * z;
            }
          }
        }
      }
      chunk_release();
      n = e;
    }
    consumer_sync();
    tr(l, 9);
    const int n4 = tid, rc = rows_cap(H, Q8W);
    float acc4[NB][4];
#pragma unroll
    for (int bb = 0; bb < NB; ++bb)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc4[bb][e] = 0.f;
    for (int n = a; n < b;) {
      const int e = down_chunk_end(n, b, rc, Q8W), nr = e - n;
      const unsigned char* st = chunk_wait();
      if (!quit && n4 < H / 4) {
        const __half* srow = reinterpret_cast<const __half*>(st + kData);
        for (int t = 0; t < nr; ++t) {
          float s[NB];
#pragma unroll
          for (int bb = 0; bb < NB; ++bb) s[bb] = act_s()[bb * 128 + (n - a) + t];
          axpy_row(st + t * rb, srow, n4, s, acc4);
        }
      }
      chunk_release();
      n = e;
    }
    if (!quit && n4 < H / 4)
      contribute(p.part_c + (size_t)cta * p.B * H, n4, acc4, tag_of(p.tag0, l, p.l0, 3));
    tr(l, 10);
  }

  // ---- tail: final norm + LM head + greedy, or the block output -----------

  __device__ __forceinline__ void tail(int a, int b) {
    const int L = p.L;
    tr(L, 0);
    float gr[kEPT];
    load_gains(p.final_norm, gr);
    const uint32_t t_out = tag_of(p.tag0, p.l1 - 1, p.l0, 4);
    reduce_slice(p.part_c, p.c_ctas, tag_of(p.tag0, p.l1 - 1, p.l0, 3),
                 p.rsum + (size_t)p.B * p.H, t_out);
    tr(L, 11);
    if (!p.run_head) {
      // the block output: every CTA reduced its slice; CTA 0 collects it
      if (cta == 0) {
        gather_norm(1, t_out, gr, 0);
        capture_rows(p.l1);
        if (p.h_out)
          for (int k = tid; k < p.B * p.H; k += kConsumers) p.h_out[k] = rs[k];
      }
      return;
    }
    gather_norm(1, t_out, gr, 0);
    tr(L, 1);
    consumer_sync();  // rs complete before CTA 0 copies it out
    capture_rows(p.l1);
    if (cta == 0 && p.h_out)
      for (int k = tid; k < p.B * p.H; k += kConsumers) p.h_out[k] = rs[k];
    const int cap = p.lm_rows;
    for (int n = a; n < b;) {
      const int e = min(b, n + cap), nr = e - n;
      if ((int)(i % p.lm_owners) == warp) {
        const unsigned char* st = chunk_wait_owned();
        if (!warp_quit()) lm_rows_mma(st, n, nr);
        __syncwarp();
        if (lane == 0 && !quit) mbar_arrive_n(&r.empty[stage], kConsumerWarps);
      }
      cursor_advance();
      n = e;
    }
    tr(L, 2);
    finish_head();
  }

  // Greedy key of logit y at vocabulary id `id`: order-preserving in y (+0 and
  // -0 equal), and on equal y the lower id is the larger key.
  __device__ __forceinline__ void fold_logit(int bb, int id, float y) {
    if (p.logits) p.logits[(size_t)bb * p.V + id] = y;
    if (isfinite(y)) {
      const uint32_t uu = (y == 0.f) ? 0u : __float_as_uint(y);
      const uint32_t ord = (uu & 0x80000000u) ? ~uu : (uu | 0x80000000u);
      const unsigned long long key = ((unsigned long long)ord << 32) | (0xffffffffu - (uint32_t)id);
#pragma unroll
      for (int b2 = 0; b2 < kMaxB; ++b2)
        if (b2 == bb && key > wbest[b2]) wbest[b2] = key;
    }
  }

  // Fold this CTA's greedy keys; the last CTA to finish writes the ids.
  __device__ __forceinline__ void finish_head() {
    if (tid < kMaxB) best[tid] = 0ull;
    consumer_sync();
#pragma unroll
    for (int bb = 0; bb < kMaxB; ++bb) {
      unsigned long long k = wbest[bb];
      for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long other = __shfl_xor_sync(0xffffffffu, k, o);
        k = other > k ? other : k;
      }
      if (lane == 0 && bb < p.B && k) atomicMax(best + bb, k);
    }
    consumer_sync();
    if (tid < p.B && !quit && best[tid]) atomicMax(p.am_key + tid, best[tid]);
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
          if (!quit) atomicCAS(p.err, 0, kErrBounds);
        } else {
          id = (int)(0xffffffffu - (uint32_t)(key & 0xffffffffu));
        }
        if (p.argmax) p.argmax[tid] = id;
      }
      if (tid == 0) atomicExch(p.am_cnt, 0u);
    }
    tr(p.L, 4);
  }
};

template <int NB, bool Q8W, int IT, int DQ>
__global__ void __launch_bounds__(kThreads, 1) decode_fused_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  Ring ring;
  ring.stages = smem;
  ring.n = p.n_stages;
  ring.full = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  ring.empty = ring.full + kMaxStages;
  // The phases read the parameters through a reference; a reference to the
  // kernel's parameter space makes every such read a long-latency generic
  // load, so they read a copy in shared memory instead.
  Params* ps = reinterpret_cast<Params*>(smem + p.off_par);
  for (int k = threadIdx.x; k < (int)(sizeof(Params) / 4); k += blockDim.x)
    reinterpret_cast<unsigned*>(ps)[k] = reinterpret_cast<const unsigned*>(&p)[k];
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.n_stages; ++s) {
      mbar_init(&ring.full[s], 1);
      mbar_init(&ring.empty[s], kConsumerWarps);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  {
    const unsigned* src = reinterpret_cast<const unsigned*>(p.layers);
    unsigned* dst = reinterpret_cast<unsigned*>(smem + p.off_tab);
    const int words = p.L * (int)sizeof(LayerDev) / 4;
    for (int k = threadIdx.x; k < words; k += blockDim.x) dst[k] = src[k];
    const unsigned* tsrc = reinterpret_cast<const unsigned*>(p.tl);
    unsigned* tdst = dst + words;
    const int twords = p.L * (int)sizeof(TLayer) / 4;
    for (int k = threadIdx.x; k < twords; k += blockDim.x) tdst[k] = tsrc[k];
    if (p.bt_in_smem) {
      int32_t* bt = reinterpret_cast<int32_t*>(smem + p.off_tab +
                                               (size_t)p.L * (sizeof(LayerDev) + sizeof(TLayer)));
      const int pps = p.kv.pages_per_seq;
      for (int k = threadIdx.x; k < p.B * pps; k += blockDim.x)
        bt[k] = p.kv.block_table[(size_t)p.seq[k / pps] * pps + k % pps];
    }
  }
  if (threadIdx.x < 16)  // the 64 zero bytes the tensor-core loads use for padding rows
    reinterpret_cast<uint32_t*>(smem + p.off_misc + 4160)[threadIdx.x] = 0u;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, c = blockIdx.x;
  const int qkvd = (p.nq + 2 * p.nkv) * p.d;
  unsigned long long* trow =
      p.trace ? p.trace + ((size_t)c * (p.L + 1) + p.L) * kTraceSlots : nullptr;
  if (trow && threadIdx.x == 0) {
    trow[12] = now_ns();
    trow[13] = clock64();
  }
  volatile unsigned int* counts =
      reinterpret_cast<volatile unsigned int*>(smem + p.off_misc + 4096 + 8 * kMaxB + 8);
  if (warp == kConsumerWarps) {
    if (lane == 0) {
      Producer pr(*ps, ring);
      for (int l = p.l0; l < p.l1 && !pr.quit; ++l) {
        int a, b;
        slice(qkvd, G, c, a, b);
        pr.phase_a(l, a, b);
        pr.phase_b(l, c, G);
        slice(p.I, G, c, a, b);
        pr.phase_c(l, a, b);
      }
      int a, b;
      slice(p.V, G, c, a, b);
      if (!pr.quit) pr.tail(a, b);
      if (trow) trow[3] = clock64();
      counts[0] = pr.i;
    }
  } else {
    Consumer<NB, Q8W, IT, DQ> cs(*ps, ring, smem);
    // `quit` is per thread (a wait that gave up), so it must not steer any
    // path that holds a consumer barrier: after an abort every thread still
    // walks all phases, with each wait returning at once and no stores.
    for (int l = p.l0; l < p.l1; ++l) {
      int a, b;
      slice(qkvd, G, c, a, b);
      cs.phase_a(l, a, b);
      cs.phase_b(l);
      slice(p.I, G, c, a, b);
      cs.phase_c(l, a, b);
    }
    int a, b;
    slice(p.V, G, c, a, b);
    cs.tail(a, b);
    if (threadIdx.x == 0) counts[1] = cs.i;
  }
  __syncthreads();
  if (trow && threadIdx.x == 0) {
    trow[14] = now_ns();
    trow[15] = clock64();
  }
  // Drain: copies issued but never consumed (after an abort) must land before
  // the CTA's shared memory is released.
  if (threadIdx.x == 0) {
    const unsigned int issued = counts[0], used = counts[1];
    const unsigned int n = (unsigned int)ring.n;
    const unsigned int first = issued > n ? issued - n : 0u;  // the newest copy of each stage
    (void)used;
    for (unsigned int k = first; k < issued; ++k) {
      const unsigned long long t0 = now_ns();
      while (!mbar_test(&ring.full[k % n], (k / n) & 1))
        if (now_ns() - t0 > 10000000ull) break;  // 10 ms
    }
  }
}

// Transposes of Wo and Wd for the fused O and down shares.
template <typename T>
__global__ void transpose_kernel(const T* __restrict__ in, int rows, int cols, T* __restrict__ out) {
  __shared__ T tile[32][33];
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int y = threadIdx.y; y < 32; y += 8) {
    const int r = r0 + y, c = c0 + threadIdx.x;
    if (r < rows && c < cols) tile[y][threadIdx.x] = in[(size_t)r * cols + c];
  }
  __syncthreads();
  for (int y = threadIdx.y; y < 32; y += 8) {
    const int c = c0 + y, r = r0 + threadIdx.x;
    if (r < rows && c < cols) out[(size_t)c * rows + r] = tile[threadIdx.x][y];
  }
}

}  // namespace fused

// ---------------------------------------------------------------------------
// Host side

namespace {

struct FusedState {
  unsigned long long* xq = nullptr;      // [kMaxB][qkv dim]
  unsigned long long* part_b = nullptr;  // [attention units][kMaxB][H]
  unsigned long long* part_c = nullptr;  // [SMs][kMaxB][H]
  unsigned long long* rsum = nullptr;    // [2][kMaxB][H]
  unsigned long long* am_key = nullptr;
  unsigned int* am_cnt = nullptr;
  int* abort_flag = nullptr;
  LayerDev* layers = nullptr;
  fused::TLayer* tl = nullptr;
  void* wo_t[64] = {};
  void* wd_t[64] = {};
  void* so_t[64] = {};
  void* sd_t[64] = {};
  uint32_t next_tag = 1;
  unsigned long long step = 0;
  int sms = 0;
  int need_stages = 1;
  bool eligible = false;
  unsigned long long wait_ns = 1000000000ull;
  int withhold = -1;
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool shape_ok(const fs_model* m) {
  const Shape& s = m->s;
  const int rep = s.nq / s.nkv;
  if (rep < 1 || rep > fused::kMaxRep) return false;
  // compiled pairs: hidden 1024 with head_dim 128, hidden 256 with head_dim 64
  if (!((s.H == 1024 && s.d == 128) || (s.H == 256 && s.d == 64))) return false;
  if (s.V >= 0x7fffffff || s.L > 64) return false;
  if (s.I % 32 || s.q_dim() % 32) return false;
  if (s.I < m->num_sms) return false;  // every CTA owns intermediate columns
  if (s.I / m->num_sms + 2 > 128) return false;  // act_s holds 128 columns per row
  if (fused::rows_cap(s.H, m->q8) < 1 || fused::pairs_cap(s.H, m->q8) < 1) return false;
  // tensor-core GEMVs: at most 48 rows per pass (QKV rows of a CTA, 2x its
  // gate/up pairs) and 32 coefficient rows (down share, O share)
  const int per = (s.I + m->num_sms - 1) / m->num_sms;
  const int qkv_per = (s.qkv_dim() + m->num_sms - 1) / m->num_sms;
  if (2 * per > 48 || qkv_per > 48 || per > 32 || rep * fused::kSlice > 32) return false;
  return true;
}

// The most chunks one phase holds at once in the ring (the bf16 phases wait
// for all their chunks before the tensor-core pass).
int chunks_needed(const Shape& s, int sms, bool q8) {
  if (q8) return 1;
  const int qd = s.nq * s.d, kvd = s.nkv * s.d, qkvd = s.qkv_dim();
  const int cap = fused::rows_cap(s.H, false), pc = fused::pairs_cap(s.H, false);
  int most = s.nq / s.nkv;
  for (int c = 0; c < sms; ++c) {
    int a, b, n = 0;
    fused::slice(qkvd, sms, c, a, b);
    for (int k = a; k < b; k = fused::qkv_chunk_end(k, b, cap, qd, kvd)) ++n;
    most = std::max(most, n);
    fused::slice(s.I, sms, c, a, b);
    most = std::max(most, (b - a + pc - 1) / pc);
    most = std::max(most, (b - a + cap - 1) / cap);
  }
  return most;
}

void state_free(FusedState* st) {
  void* bufs[] = {st->xq,     st->part_b,     st->part_c, st->rsum,  st->am_key,
                  st->am_cnt, st->abort_flag, st->layers, st->tl};
  for (void* b : bufs)
    if (b) cudaFree(b);
  for (int l = 0; l < 64; ++l) {
    if (st->wo_t[l]) cudaFree(st->wo_t[l]);
    if (st->wd_t[l]) cudaFree(st->wd_t[l]);
    if (st->so_t[l]) cudaFree(st->so_t[l]);
    if (st->sd_t[l]) cudaFree(st->sd_t[l]);
  }
}

template <typename T>
void launch_transpose(const void* in, int rows, int cols, void* out) {
  dim3 grid((cols + 31) / 32, (rows + 31) / 32), block(32, 8);
  count_launches();
  fused::transpose_kernel<T><<<grid, block>>>(static_cast<const T*>(in), rows, cols,
                                              static_cast<T*>(out));
}

}  // namespace

bool fused_eligible(const fs_model* m) {
  const FusedState* st = static_cast<const FusedState*>(m->extras);
  return st && st->eligible;
}

fs_status fused_init(fs_model* m) {
  FusedState* st = new FusedState();
  m->extras = st;
  st->sms = m->num_sms;
  st->eligible = shape_ok(m);
  if (!st->eligible) return FS_OK;
  const Shape& s = m->s;
  st->need_stages = chunks_needed(s, m->num_sms, m->q8);
  auto alloc = [&](void** p, size_t bytes) {
    if (cudaMalloc(p, bytes) != cudaSuccess) {
      cudaGetLastError();
      *p = nullptr;
      return false;
    }
    cudaMemset(*p, 0, bytes);
    return true;
  };
  const size_t w = sizeof(unsigned long long);
  // per set: arrival counters [2L][kMaxCopies], then the accumulator words
  const size_t units = (size_t)s.nkv * (s.d / fused::kSlice);
  const size_t rows = (size_t)fused::kMaxB * s.H;
  bool ok = alloc((void**)&st->xq, (size_t)fused::kMaxB * s.qkv_dim() * w) &&
            alloc((void**)&st->part_b, units * rows * w) &&
            alloc((void**)&st->part_c, (size_t)st->sms * rows * w) &&
            alloc((void**)&st->rsum, 2 * rows * w) &&
            alloc((void**)&st->am_key, (size_t)fused::kMaxB * w) &&
            alloc((void**)&st->am_cnt, 64) && alloc((void**)&st->abort_flag, 64) &&
            alloc((void**)&st->layers, (size_t)s.L * sizeof(LayerDev)) &&
            alloc((void**)&st->tl, (size_t)s.L * sizeof(fused::TLayer));
  // Transposed Wo [H][nq d] -> [nq d][H] and Wd [H][I] -> [I][H] (codes and
  // scales for Q8_0), library-owned.
  std::vector<fused::TLayer> tl(s.L);
  for (int l = 0; ok && l < s.L; ++l) {
    const LayerDev& Lw = m->layers[l];
    const size_t eb = m->q8 ? 1 : 2;
    ok = alloc(&st->wo_t[l], (size_t)s.q_dim() * s.H * eb) &&
         alloc(&st->wd_t[l], (size_t)s.I * s.H * eb);
    if (ok && m->q8)
      ok = alloc(&st->so_t[l], (size_t)(s.q_dim() / 32) * s.H * 2) &&
           alloc(&st->sd_t[l], (size_t)(s.I / 32) * s.H * 2);
    if (!ok) break;
    if (m->q8) {
      launch_transpose<int8_t>(Lw.w[kWo], s.H, s.q_dim(), st->wo_t[l]);
      launch_transpose<int8_t>(Lw.w[kWd], s.H, s.I, st->wd_t[l]);
      launch_transpose<unsigned short>(Lw.s[kWo], s.H, s.q_dim() / 32, st->so_t[l]);
      launch_transpose<unsigned short>(Lw.s[kWd], s.H, s.I / 32, st->sd_t[l]);
    } else {
      launch_transpose<unsigned short>(Lw.w[kWo], s.H, s.q_dim(), st->wo_t[l]);
      launch_transpose<unsigned short>(Lw.w[kWd], s.H, s.I, st->wd_t[l]);
    }
    tl[l] = fused::TLayer{st->wo_t[l], static_cast<const __half*>(st->so_t[l]), st->wd_t[l],
                          static_cast<const __half*>(st->sd_t[l])};
  }
  if (!ok || cudaGetLastError() != cudaSuccess) {
    state_free(st);
    delete st;
    m->extras = nullptr;
    set_error("out of device memory for the decode kernel's buffers");
    return FS_ERR_OOM;
  }
  cudaMemcpy(st->layers, m->layers.data(), (size_t)s.L * sizeof(LayerDev), cudaMemcpyHostToDevice);
  cudaMemcpy(st->tl, tl.data(), (size_t)s.L * sizeof(fused::TLayer), cudaMemcpyHostToDevice);
  const void* kernels[] = {
      (const void*)fused::decode_fused_kernel<1, false, 4, 32>, (const void*)fused::decode_fused_kernel<1, true, 4, 32>,
      (const void*)fused::decode_fused_kernel<4, false, 4, 32>, (const void*)fused::decode_fused_kernel<4, true, 4, 32>,
      (const void*)fused::decode_fused_kernel<1, false, 1, 16>, (const void*)fused::decode_fused_kernel<1, true, 1, 16>,
      (const void*)fused::decode_fused_kernel<4, false, 1, 16>, (const void*)fused::decode_fused_kernel<4, true, 1, 16>};
  for (const void* k : kernels)
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
  return FS_OK;
}

void fused_release(fs_model* m) {
  FusedState* st = static_cast<FusedState*>(m->extras);
  if (!st) return;
  state_free(st);
  delete st;
  m->extras = nullptr;
}

// Clears the exchange state after a step was aborted (device error seen).
void fused_reset(fs_model* m) {
  FusedState* st = static_cast<FusedState*>(m->extras);
  if (!st || !st->eligible) return;
  cudaDeviceSynchronize();
  cudaMemset(st->am_key, 0, (size_t)fused::kMaxB * sizeof(unsigned long long));
  cudaMemset(st->am_cnt, 0, 64);
  cudaMemset(st->abort_flag, 0, 64);
  st->next_tag += 1u << 20;  // every tag in flight is now stale
}

void fused_debug_wait(fs_model* m, unsigned long long wait_ns, int withhold_layer) {
  FusedState* st = static_cast<FusedState*>(m->extras);
  if (!st) return;
  st->wait_ns = wait_ns;
  st->withhold = withhold_layer;
}

fs_status decode_fused(fs_model* m, const fs_kv* kv, const RowMap& map, int B, const int32_t* tok,
                       const float* h_in, float* h_out, int l0, int l1, bool run_head,
                       float* logits, int32_t* argmax, cudaStream_t stream) {
  FusedState* st = static_cast<FusedState*>(m->extras);
  if (!st || !st->eligible || B > fused::kMaxB || B < 1) return FS_ERR_UNSUPPORTED;
  const Shape& s = m->s;
  fused::Params p{};
  p.L = s.L; p.H = s.H; p.nq = s.nq; p.nkv = s.nkv; p.d = s.d; p.I = s.I; p.V = s.V;
  p.eps = s.eps;
  p.q8 = m->q8 ? 1 : 0;
  p.layers = st->layers;
  p.tl = st->tl;
  p.embed = m->embed;
  p.final_norm = m->final_norm;
  p.rope = m->rope;
  p.kv = kv_view(kv);
  p.B = B;
  for (int b = 0; b < B; ++b) {
    const RowInfo ri = map.get(b);
    p.seq[b] = ri.seq;
    p.pos[b] = ri.pos;
  }
  p.tokens = tok;
  p.xq = st->xq;
  p.part_b = st->part_b;
  p.part_c = st->part_c;
  p.rsum = st->rsum;
  p.n_units = s.nkv * (s.d / fused::kSlice);
  p.c_ctas = std::min(s.I, st->sms);
  p.l0 = l0;
  p.l1 = l1;
  p.h_in = h_in;
  p.h_out = h_out;
  p.run_head = run_head ? 1 : 0;
  p.logits = logits;
  p.argmax = argmax;
  p.am_key = st->am_key;
  p.am_cnt = st->am_cnt;
  p.capture = m->capture;
  p.capture_stride = m->capture_max_rows;
  p.err = m->err;
  p.abort_flag = st->abort_flag;
  p.wait_ns = st->wait_ns;
  p.withhold_layer = st->withhold;
  st->withhold = -1;  // one-shot
  p.trace = m->trace;
  m->trace = nullptr;  // one-shot
  if (st->next_tag > 0xF0000000u) {
    // wrap: clear the tags so the numbering can restart
    cudaStreamSynchronize(stream);
    const size_t w = sizeof(unsigned long long), rows = (size_t)fused::kMaxB * s.H;
    cudaMemsetAsync(st->xq, 0, (size_t)fused::kMaxB * s.qkv_dim() * w, stream);
    cudaMemsetAsync(st->part_b, 0, (size_t)p.n_units * rows * w, stream);
    cudaMemsetAsync(st->part_c, 0, (size_t)st->sms * rows * w, stream);
    cudaMemsetAsync(st->rsum, 0, 2 * rows * w, stream);
    st->next_tag = 1;
  }
  p.tag0 = st->next_tag;
  st->next_tag += 5u * (uint32_t)(l1 - l0) + 1u;
  // shared memory carve-up
  const size_t rows_bytes = align_up((size_t)B * s.H * 4, 128);
  const size_t zs_bytes = m->q8 ? 2 * rows_bytes : 0;
  const size_t zt_bytes = align_up((size_t)2 * 2 * B * (s.H + 8) * 2, 128);
  const size_t misc = 5120;
  const size_t attn = align_up((size_t)(fused::kMaxRep * 128 + 256 +
                                        fused::kConsumerWarps * fused::kMaxRep * 10) * 4, 128);
  const size_t tab_ptrs = (size_t)s.L * (sizeof(LayerDev) + sizeof(fused::TLayer));
  const size_t bt_bytes = (size_t)B * kv->pages_per_seq * sizeof(int32_t);
  const bool bt_smem = bt_bytes <= 8192;
  const size_t tab = align_up(tab_ptrs + (bt_smem ? bt_bytes : 0), 128);
  const size_t bars = 2 * fused::kMaxStages * 8;
  // the slice reducer: [contributors][slice] values + 4 partial sums per element
  const int emax = (B * s.H + st->sms - 1) / st->sms;
  // ... and the tensor-core partial sums: 3 row tiles x H/128 k-blocks x 64
  const size_t red = align_up(std::max((size_t)(std::max(p.n_units, st->sms) + 4) * emax * 4,
                                       (size_t)3 * (s.H / 128) * 64 * 4),
                              128);
  const size_t par = align_up(sizeof(fused::Params), 128);
  const size_t fixed = rows_bytes + zs_bytes + zt_bytes + misc + attn + tab + bars + red + par;
  const size_t budget = 232448;
  p.stage_bytes = m->q8 ? fused::kStageQ8 : fused::kStageBf16;
  int n_stages = (int)((budget - fixed) / (size_t)p.stage_bytes);
  n_stages = std::min(n_stages, fused::kMaxStages);
  if (n_stages < 4 || n_stages < st->need_stages) return FS_ERR_UNSUPPORTED;
  size_t off = (size_t)n_stages * p.stage_bytes;
  p.off_r = (int)off; off += rows_bytes;
  p.off_z = (int)off; off += zs_bytes;
  p.off_zt = (int)off; off += zt_bytes;
  p.off_misc = (int)off; off += misc;
  p.off_attn = (int)off; off += attn;
  p.off_bar = (int)off; off += bars;
  p.off_tab = (int)off; off += tab;
  p.off_red = (int)off; off += red;
  p.off_par = (int)off; off += par;
  p.bt_in_smem = bt_smem ? 1 : 0;
  p.n_stages = n_stages;
  // A warp that consumes only every lm_owners-th chunk tests the release of
  // the chunk a ring earlier before the chunk itself; that test is
  // unambiguous when the ring holds at least lm_owners stages.
  p.lm_owners = std::min(fused::kConsumerWarps, n_stages);
  p.lm_rows = std::min(8, fused::rows_cap(s.H, false));
  void* args[] = {&p};
  const bool h1k = s.H == 1024;
  const void* fn;
  if (B == 1)
    fn = m->q8 ? (h1k ? (const void*)fused::decode_fused_kernel<1, true, 4, 32>
                      : (const void*)fused::decode_fused_kernel<1, true, 1, 16>)
               : (h1k ? (const void*)fused::decode_fused_kernel<1, false, 4, 32>
                      : (const void*)fused::decode_fused_kernel<1, false, 1, 16>);
  else
    fn = m->q8 ? (h1k ? (const void*)fused::decode_fused_kernel<4, true, 4, 32>
                      : (const void*)fused::decode_fused_kernel<4, true, 1, 16>)
               : (h1k ? (const void*)fused::decode_fused_kernel<4, false, 4, 32>
                      : (const void*)fused::decode_fused_kernel<4, false, 1, 16>);
  count_launches();
  cudaError_t e = cudaLaunchCooperativeKernel(fn, dim3(st->sms), dim3(fused::kThreads), args, off,
                                              stream);
  if (e != cudaSuccess) {
    set_error(std::string("decode kernel launch failed: ") + cudaGetErrorString(e));
    return FS_ERR_CUDA;
  }
  ++st->step;
  return FS_OK;
}

}  // namespace fs
