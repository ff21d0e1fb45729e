// Persistent decode forward on thread-block clusters, for batches of 1..4
// sequences with bf16 weights: one launch of n_kv_heads clusters of 16 CTAs
// runs every block, the final norm, the tied LM head and the greedy argmax of
// one decode step.
//
// Cluster g owns kv head g and everything that only depends on it; CTA r of
// the cluster (rank r) owns a sixteenth of each of its products:
//   A  RMSNorm of the block input (every CTA, whole rows), then the cluster's
//      (rep + 2) * d rows of Wq|Wk|Wv (rep query heads, k and v of head g):
//      CTA r computes 1/16 of them. The raw rows go to every CTA of the
//      cluster, which all apply the per-head q/k RMSNorm and RoPE; rank 0
//      appends k and v to the cache.
//   B  attention of the rep query heads over the cache: the keys are split
//      into 16 contiguous ranges, one per CTA (rank 0 also takes the new
//      key); each CTA sends its softmax state (max, sum, unnormalised output)
//      of each output element to the CTA that owns it (1/16 of the rep * d
//      outputs), which merges the 16 states; the merged outputs go to every
//      CTA. The output projection is split by rows: CTA r multiplies rows
//      [r H/16, (r+1) H/16) of the cluster's rep * d columns of Wo by the
//      cluster's outputs; the result is the cluster's share of those rows.
//   C  RMSNorm of the residual after attention, then the cluster's I / n_kv
//      intermediate columns (CTA r: 1/16 of them) of Wg and Wu, SwiGLU; the
//      activations go to every CTA of the cluster; the down projection is
//      split by rows like the output projection.
// Inside a cluster, data moves through distributed shared memory: each
// exchange is a set of st.async stores into the destination CTAs' shared
// memory that complete on the destination's transaction barrier; no fence
// and no extra arrival is needed. Across clusters there are two hand-offs per
// block: the O-projection shares (after B) and the down-projection shares
// (after C), as 64-bit words (fp32 value | tag) in a slot per cluster; CTA r
// of every cluster sums slice r of the n_kv slots in a fixed order (so the
// result is reproducible bit for bit), adds the residual and sends the slice
// to the whole cluster.
//
// Weight stream: at model creation the weights every CTA multiplies in a
// block are packed into one contiguous image per (block, CTA), in the order
// the CTA uses them, cut into chunks of whole rows that each fill one ring
// stage, with the 16-byte units of row j stored at unit index u ^ (j mod 8)
// (so the tensor-core operand loads of 8 rows hit 8 different bank groups);
// Q8_0 chunks hold the rows' int8 codes followed by their fp16 scales. A
// producer warp copies each chunk with one bulk copy, then the CTA's K/V
// ranges and, for the LM head, runs of whole embedding rows, into a ring of
// shared-memory stages, running ahead across phases and blocks. The skinny
// products run on the tensor cores (mma.sync m16n8k16, bf16 in, fp32
// accumulate) with the activation as two bf16 terms (hi + lo), so each
// product keeps about 16 bits of the fp32 activation; Q8_0 codes become bf16
// exactly and each 32-wide block's product is scaled in fp32.
//
// Every wait is bounded by %globaltimer; on timeout the CTA records
// kErrTimeout and raises the abort flag that every wait checks; all CTAs then
// still walk every exchange (with stale values and no global stores), so each
// exchange completes and no CTA leaves while a peer may write into it.
#include <algorithm>

#include "runtime.h"

namespace fs {
namespace clus {

constexpr int kMaxCS = 16;  // CTAs per cluster (16, or 8 where 16-CTA clusters do not all fit)
constexpr int kConsumerWarps = 11;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;  // + producer warp
constexpr int kMaxB = 4;
constexpr int kStage = 17408;  // ring stage: 16 Q8_0 rows of K = 1024 with their scales
constexpr int kMaxStages = 14;
constexpr int kTraceSlots = 16;
constexpr int kMaxRows = 128;  // rows of one tensor-core pass
constexpr int kMaxH = 1024;

// How the work of a block is split. Clusters: `split` per kv head, each
// taking rep / split of the head's query heads (and the head's k and v
// rows, so with split > 1 the k and v projections run in every cluster of
// the head); CTAs: `cs` per cluster.
struct Geo {
  int cs, split, ncl, repc;
  int nA;      // QKV rows per CTA: (repc + 2) d / cs
  int nO;      // O and down rows per CTA: H / cs
  int nc;      // intermediate columns per CTA: I / (ncl cs)
  int Kc;      // intermediate columns per cluster (the down product's K): I / ncl
  int RDc;     // attention outputs per cluster: repc d (the O product's K)
  int F;       // attention outputs merged by one CTA: RDc / cs
  int n[4], K[4];  // rows and K of the four weight phases
};

struct Params {
  int L, H, nq, nkv, d, I, V;
  float eps;
  Geo geo;
  const LayerDev* layers;
  const __nv_bfloat16* embed;
  const __nv_bfloat16* final_norm;
  const float2* rope;
  KVView kv;
  int B;
  int seq[kMaxB];
  int pos[kMaxB];
  const int32_t* tokens;
  unsigned long long* po;  // [clusters][kMaxB][H] O-projection shares (tagged)
  unsigned long long* pd;  // [clusters][kMaxB][H] down-projection shares (tagged)
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
  int withhold_layer;  // debug: the O-projection shares of this layer are never published
  unsigned long long* trace;
  int n_stages;
  int lm_owners, lm_rows;
  int bt_in_smem;
  int off_par;  // a copy of these parameters in shared memory (see the kernel)
  int q8;
  const unsigned char* packed;  // [L][clusters][cs] per-CTA weight images of stream_bytes each
  int stream_bytes;
  int pofs[4];                  // offsets of the four phases in an image
  // shared-memory carve-up (byte offsets)
  int off_ha, off_hm, off_zt, off_zo, off_za, off_raw, off_q, off_kv, off_att, off_cmb, off_act,
      off_ssc, off_ys, off_red, off_ss, off_misc, off_bar, off_tab;
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
__device__ __forceinline__ void mbar_arrive_n(uint64_t* bar, uint32_t n) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(su32(bar)), "r"(n) : "memory");
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
// The same test with acquire at cluster scope: the data other CTAs stored
// with st.async before completing the phase are visible after it.
__device__ __forceinline__ bool mbar_test_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
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
// Bulk copy global -> this CTA's shared memory (never another CTA's).
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
__device__ __forceinline__ uint32_t word_tag(unsigned long long w) { return (uint32_t)(w >> 32); }
__device__ __forceinline__ float word_value(unsigned long long w) {
  return __uint_as_float((uint32_t)w);
}
__device__ __forceinline__ unsigned long long now_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory");
}
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
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
// 4 bytes into another CTA's shared memory, completing on its barrier.
__device__ __forceinline__ void st_async(uint32_t raddr, uint32_t v, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(
                   raddr),
               "r"(v), "r"(rbar)
               : "memory");
}
// Every thread of every CTA of the cluster (the warp converged first).
__device__ __forceinline__ void cluster_sync_all() {
  __syncwarp();
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
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
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}
__device__ __forceinline__ float lds_half(uint32_t addr) {
  unsigned short h;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(h) : "r"(addr));
  return __half2float(__ushort_as_half(h));
}
// Bytes 2i, 2i + 1 of w as int8 values, converted exactly to a bf16 pair
// (byte 2i in the low half).
__device__ __forceinline__ uint32_t i8x2_bf16(uint32_t w, int i) {
  const int lo = (int)(w << (24 - 16 * i)) >> 24, hi = (int)(w << (16 - 16 * i)) >> 24;
  const __nv_bfloat162 v = __floats2bfloat162_rn((float)lo, (float)hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}
// fp32 -> (hi, lo) bf16 terms, hi + lo = x to about 16 bits.
__device__ __forceinline__ void split_bf16(float x, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}
__device__ __forceinline__ uint32_t pack2(__nv_bfloat16 a, __nv_bfloat16 b) {
  return (uint32_t)__bfloat16_as_ushort(a) | ((uint32_t)__bfloat16_as_ushort(b) << 16);
}

__host__ __device__ inline void slice(int N, int G, int c, int& a, int& b) {
  a = (int)((long long)N * c / G);
  b = (int)((long long)N * (c + 1) / G);
}
// The weight phases of a block, in the order a CTA uses them: its rows of
// Wq|Wk|Wv (A), of Wo (O), of Wg then Wu (GU) and of Wd (D).
enum { kPA = 0, kPO, kPGU, kPD, kPhases };
// Bytes of one packed row of K weights (Q8_0: codes + scales), rows per
// chunk (a multiple of 8 that fits a stage) and bytes of a chunk of nr rows.
__host__ __device__ inline int row_bytes(int K, bool q8) { return q8 ? K + K / 16 : 2 * K; }
__host__ __device__ inline int cap_rows(int K, bool q8) {
  const int c = kStage / row_bytes(K, q8);
  return c >= 8 ? (c & ~7) : c;
}
__host__ __device__ inline int chunk_bytes(int nr, int K, bool q8) {
  return (nr * row_bytes(K, q8) + 15) & ~15;
}
__host__ __device__ inline int phase_bytes(int n, int K, bool q8) {
  const int cap = cap_rows(K, q8), full = n / cap, rest = n - full * cap;
  return full * chunk_bytes(cap, K, q8) + (rest ? chunk_bytes(rest, K, q8) : 0);
}

// Tag of hand-off k of block l: 0 O-projection shares, 1 down-projection shares.
__host__ __device__ __forceinline__ uint32_t tag_of(uint32_t tag0, int l, int l0, int k) {
  return tag0 + 2u * (uint32_t)(l - l0) + (uint32_t)k;
}

struct Ring {
  unsigned char* stages;
  uint64_t* full;
  uint64_t* empty;
  int n;
};

__device__ __forceinline__ const LayerDev& layer_s(const Params& p, int l) {
  extern __shared__ __align__(1024) unsigned char smem_base[];
  return reinterpret_cast<const LayerDev*>(smem_base + p.off_tab)[l];
}
__device__ __forceinline__ size_t kv_off(const Params& p, int layer, int b, int pos, int g) {
  extern __shared__ __align__(1024) unsigned char smem_base[];
  int page;
  if (p.bt_in_smem) {
    const int32_t* bt =
        reinterpret_cast<const int32_t*>(smem_base + p.off_tab + (size_t)p.L * sizeof(LayerDev));
    page = bt[b * p.kv.pages_per_seq + pos / kPage];
  } else {
    page = p.kv.block_table[(size_t)p.seq[b] * p.kv.pages_per_seq + pos / kPage];
  }
  return (size_t)layer * p.kv.layer_elems() +
         (((size_t)page * p.kv.n_kv_heads + g) * kPage + (pos % kPage)) * p.kv.head_dim;
}

__host__ __device__ inline Geo make_geo(int H, int nq, int nkv, int d, int I, int cs, int split) {
  Geo g{};
  g.cs = cs;
  g.split = split;
  g.ncl = nkv * split;
  g.repc = nq / nkv / split;
  g.nA = (g.repc + 2) * d / cs;
  g.nO = H / cs;
  g.nc = I / (g.ncl * cs);
  g.Kc = I / g.ncl;
  g.RDc = g.repc * d;
  g.F = g.RDc / cs;
  g.n[kPA] = g.nA;
  g.K[kPA] = H;
  g.n[kPO] = g.nO;
  g.K[kPO] = g.RDc;
  g.n[kPGU] = 2 * g.nc;
  g.K[kPGU] = H;
  g.n[kPD] = g.nO;
  g.K[kPD] = g.Kc;
  return g;
}
// The 16-byte unit u of packed row j sits at unit u ^ (j mod 8), within each
// whole group of 8 units (a row's last partial group stays in place).
__host__ __device__ inline int swz(int u, int j, int units) {
  return (u | 7) < units ? (u ^ (j & 7)) : u;
}

// ---------------------------------------------------------------------------
// Out-of-line waiting loops. They are free functions taking plain values, not
// members: a member function that is not inlined takes the object's address,
// which moves the whole object (ring cursor, flags, ...) to the stack, and
// with shared memory taking most of L1 every member access then waits on
// memory.

// Warp-wide wait until bar1 (if not null) shows phase par1 and bar0 phase
// par0, or the wait runs out; true if it ran out. `quit`: this lane gave up.
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
// when the wait runs out (the last value read is returned).
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
  unsigned int i = 0;  // chunks issued
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
    return r.stages + (size_t)s * kStage;
  }
  __device__ __forceinline__ uint64_t* bar() { return &r.full[stage]; }
  __device__ __forceinline__ void advance() {
    ++i;
    if (++stage == r.n) {
      stage = 0;
      parity ^= 1u;
    }
  }
  // The n packed rows of K weights of one phase, one bulk copy per chunk.
  __device__ void weights(const unsigned char* src, int n, int K) {
    const bool q8 = p.q8 != 0;
    const int cap = cap_rows(K, q8);
    for (int j0 = 0; j0 < n && !quit; j0 += cap) {
      const uint32_t bytes = (uint32_t)chunk_bytes(min(cap, n - j0), K, q8);
      unsigned char* st = acquire(bytes);
      if (!st) return;
      bulk_load(st, src, bytes, bar(), policy);
      advance();
      src += bytes;
    }
  }

  __device__ void layer(int l, int c, int g, int rk) {
    const Geo& G = p.geo;
    const unsigned char* img =
        p.packed + ((size_t)(l * G.ncl + c) * G.cs + rk) * (size_t)p.stream_bytes;
    weights(img + p.pofs[kPA], G.n[kPA], G.K[kPA]);
    // B: the CTA's key range of each batch row, K then V per page segment
    const int d = p.d;
    for (int b = 0; b < p.B && !quit; ++b) {
      int k0, k1;
      slice(p.pos[b], G.cs, rk, k0, k1);
      for (int j0 = k0; j0 < k1 && !quit;) {
        const int je = min(k1, (j0 / kPage + 1) * kPage), nk = je - j0;
        const size_t off = kv_off(p, l, b, j0, g);
        unsigned char* st = acquire(nk * d * 2);
        if (!st) return;
        bulk_load(st, p.kv.k + off, nk * d * 2, bar(), policy);
        advance();
        st = acquire(nk * d * 2);
        if (!st) return;
        bulk_load(st, p.kv.v + off, nk * d * 2, bar(), policy);
        advance();
        j0 = je;
      }
    }
    weights(img + p.pofs[kPO], G.n[kPO], G.K[kPO]);
    weights(img + p.pofs[kPGU], G.n[kPGU], G.K[kPGU]);
    weights(img + p.pofs[kPD], G.n[kPD], G.K[kPD]);
  }

  // LM head: runs of lm_rows whole embedding rows, one bulk copy each.
  __device__ void tail(int a, int b) {
    if (!p.run_head) return;
    const int cap = p.lm_rows;
    for (int n = a; n < b && !quit;) {
      const int e = min(b, n + cap), nr = e - n;
      unsigned char* st = acquire(nr * 2 * p.H);
      if (!st) return;
      bulk_load(st, p.embed + (size_t)n * p.H, nr * 2 * p.H, bar(), policy);
      advance();
      n = e;
    }
  }
};

// ---------------------------------------------------------------------------
// Consumers

template <int NB, bool Q8>
struct Consumer {
  const Params& p;
  Ring r;
  unsigned char* sm;
  unsigned int i = 0;  // chunks consumed
  int stage = 0;
  uint32_t parity = 0;
  bool quit = false;
  unsigned int xk = 0;  // exchanges done
  int cur_layer = 0;    // for trace stamps
  unsigned int grp = 0;  // owner-mode chunk groups so far (the owner of the next one is grp % W)
  int tid, warp, lane, cta, cl, g, hs, rk, G;
  float inv[NB];
  unsigned long long wbest[kMaxB] = {0ull, 0ull, 0ull, 0ull};
  static constexpr int kEPT = (NB * kMaxH + kConsumers - 1) / kConsumers;

  __device__ Consumer(const Params& pp, Ring rr, unsigned char* s) : p(pp), r(rr), sm(s) {
    tid = threadIdx.x;
    warp = tid >> 5;
    lane = tid & 31;
    cta = blockIdx.x;
    G = gridDim.x;
    rk = (int)cluster_rank();
    cl = cta / p.geo.cs;      // cluster
    g = cl / p.geo.split;     // its kv head
    hs = cl % p.geo.split;    // its share of the head's query heads
  }

  // ---- shared-memory regions ---------------------------------------------
  __device__ float* ha() { return reinterpret_cast<float*>(sm + p.off_ha); }  // [B][H] block input
  __device__ float* hm() { return reinterpret_cast<float*>(sm + p.off_hm); }  // [B][H] after attention
  __device__ __nv_bfloat16* zt() { return reinterpret_cast<__nv_bfloat16*>(sm + p.off_zt); }
  __device__ int zt_stride() const { return p.H + 8; }  // [2B][H + 8]: hi, lo rows of each batch row
  __device__ __nv_bfloat16* zo() { return reinterpret_cast<__nv_bfloat16*>(sm + p.off_zo); }
  __device__ int zo_stride() const { return p.geo.RDc + 8; }
  __device__ __nv_bfloat16* za() { return reinterpret_cast<__nv_bfloat16*>(sm + p.off_za); }
  __device__ int za_stride() const { return p.geo.Kc + 8; }
  __device__ float* raw() { return reinterpret_cast<float*>(sm + p.off_raw); }  // [B][(repc+2)d]
  __device__ float* qs() { return reinterpret_cast<float*>(sm + p.off_q); }     // [B][repc][d]
  __device__ __nv_bfloat16* kcur() { return reinterpret_cast<__nv_bfloat16*>(sm + p.off_kv); }
  __device__ __nv_bfloat16* vcur() { return kcur() + kMaxB * p.d; }
  __device__ float* att() { return reinterpret_cast<float*>(sm + p.off_att); }  // [cs][kMaxB][2 + F]
  __device__ float* cmb() { return reinterpret_cast<float*>(sm + p.off_cmb); }  // [B][F]
  __device__ float* act() { return reinterpret_cast<float*>(sm + p.off_act); }  // [B][nc]
  __device__ float* ssc() { return reinterpret_cast<float*>(sm + p.off_ssc); }  // [rep][64] + run state
  __device__ float* ys() { return reinterpret_cast<float*>(sm + p.off_ys); }    // [128][4]
  __device__ float* red() { return reinterpret_cast<float*>(sm + p.off_red); }  // exchange sums
  __device__ float* ssp() { return reinterpret_cast<float*>(sm + p.off_ss); }   // [11][kMaxB]
  // misc (bytes): zero bytes 0..64, greedy keys 64..96, flag 96, counts 104.
  __device__ uint32_t zero_addr() { return su32(sm + p.off_misc); }  // 64 zero bytes
  __device__ unsigned long long* best() {
    return reinterpret_cast<unsigned long long*>(sm + p.off_misc + 64);
  }
  __device__ int* flag() { return reinterpret_cast<int*>(sm + p.off_misc + 96); }
  __device__ uint64_t* xbar() { return r.empty + kMaxStages; }  // [2] exchange barriers

  // ---- ring --------------------------------------------------------------
  __device__ __forceinline__ uint32_t stage_addr(int ahead) const {
    int s = stage + ahead;
    if (s >= r.n) s -= r.n;
    return su32(r.stages + (size_t)s * kStage);
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
  // warp has not released (every chunk before it waited for by this warp).
  //
  // The common case (the chunk is in) is inline; the waiting loop is not, so
  // loops over chunks make no function call (calls spill registers to the
  // stack, and with shared memory taking most of L1 those spills go to L2).
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
    return r.stages + (size_t)s * kStage;
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
  // Owner-mode wait of the LM head (this warp alone consumes the chunk): the
  // release of the chunk a ring earlier in the same stage, then the chunk.
  __device__ __forceinline__ const unsigned char* chunk_wait_owned(int ahead = 0) {
    int s = stage + ahead;
    uint32_t par = parity;
    if (s >= r.n) {
      s -= r.n;
      par ^= 1u;
    }
    if (!__all_sync(0xffffffffu, quit || (mbar_test(&r.empty[s], par ^ 1u) &&
                                          mbar_test(&r.full[s], par))) &&
        warp_wait_slow(&r.full[s], par, &r.empty[s], par ^ 1u, quit, p.wait_ns, p.abort_flag))
      give_up();
    return r.stages + (size_t)s * kStage;
  }
  // Owner-mode release of the chunk `ahead` places after the cursor.
  __device__ __forceinline__ void chunk_release_owned(int ahead) {
    int s = stage + ahead;
    if (s >= r.n) s -= r.n;
    __syncwarp();
    if (lane == 0 && !quit) mbar_arrive_n(&r.empty[s], kConsumerWarps);
  }

  // ---- cluster exchanges ---------------------------------------------------
  // Exchange xk uses barrier xk % 2 in phase (xk / 2) % 2. A CTA sends the
  // data of exchange xk + 1 only after its own exchange xk completed, which
  // needed every peer's data of exchange xk: so no peer is ever two exchanges
  // ahead, and the two barriers never see bytes of a later phase.
  __device__ __forceinline__ void xarm(uint32_t bytes) {
    if (tid == 0) mbar_expect_tx(&xbar()[xk & 1], bytes);
  }
  __device__ __forceinline__ void xsend(const void* local_dst, int dest, uint32_t v) {
    st_async(mapa(su32(local_dst), (uint32_t)dest), v, mapa(su32(&xbar()[xk & 1]), (uint32_t)dest));
  }
  __device__ __forceinline__ void xwait() {
    uint64_t* bar = &xbar()[xk & 1];
    const uint32_t par = (xk >> 1) & 1u;
    unsigned long long t0 = 0;
    int spins = 0;
    while (!mbar_test_cluster(bar, par)) {
      __nanosleep(32);
      if (quit) break;
      if ((++spins & 15) == 0) {
        if (wait_expired(t0, p.wait_ns, p.abort_flag)) {
          give_up();
          break;
        }
      }
    }
    ++xk;
    consumer_sync();  // the received data are read by every thread after this
  }

  // Polls one tagged word until its tag is `want` (bounded); x: the value
  // already loaded.
  __device__ __forceinline__ unsigned long long poll_word(const unsigned long long* w,
                                                          unsigned long long x, uint32_t want) {
    if (word_tag(x) == want || quit) return x;
    bool gave_up = false;
    x = poll_slow(w, want, p.wait_ns, p.abort_flag, &gave_up);
    if (gave_up) give_up();
    return x;
  }

  // dst = base + sum over clusters of the tagged shares src[c][B][H], for the
  // whole rows: this CTA sums its slice (elements [rk E, (rk+1) E) of each
  // row, E = H / cs, clusters in order) and sends it to every CTA of the
  // cluster. The slice of cluster c is what rank rk of cluster c published.
  // One thread per cluster first waits for that CTA's last word, so only a
  // few threads poll while the shares are still coming; then every thread
  // loads its words once (a word still stale is polled on its own). Ends
  // with the exchange complete.
  __device__ __forceinline__ void exchange_sum(const unsigned long long* src, uint32_t tag,
                                            const float* base, float* dst) {
    const int H = p.H, E = H / p.geo.cs, e0 = rk * E, n = p.B * E, total = p.geo.ncl * n;
    float* buf = red();
    float* sums = buf + total;
    if (tid < p.geo.ncl) {
      const unsigned long long* last = src + ((size_t)tid * kMaxB + p.B - 1) * H + e0 + E - 1;
      poll_word(last, ld_word(last), tag);
    }
    consumer_sync();
    for (int f0 = tid; f0 < total; f0 += 4 * kConsumers) {
      unsigned long long w[4];
      const unsigned long long* ptr[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int f = f0 + u * kConsumers;
        const int c = f / n, v = f % n;
        ptr[u] = f < total ? src + ((size_t)c * kMaxB + v / E) * H + e0 + v % E : src;
        w[u] = f < total ? ld_word(ptr[u]) : 0ull;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int f = f0 + u * kConsumers;
        if (f < total) buf[f] = word_value(poll_word(ptr[u], w[u], tag));
      }
    }
    consumer_sync();
    for (int v = tid; v < n; v += kConsumers) {
      float s = 0.f;
      for (int c = 0; c < p.geo.ncl; ++c) s += buf[c * n + v];
      sums[v] = base[(v / E) * H + e0 + v % E] + s;
    }
    consumer_sync();
    xarm((uint32_t)(p.B * H * 4));
    for (int w = tid; w < n * p.geo.cs; w += kConsumers) {
      const int dest = w / n, v = w % n;
      xsend(dst + (v / E) * H + e0 + v % E, dest, __float_as_uint(sums[v]));
    }
    xwait();
  }

  // The block input of the first block: embedding rows of the tokens (or
  // h_in), whole rows, computed by every CTA. Ends on a barrier.
  __device__ __forceinline__ void first_input() {
    const int H = p.H;
    for (int k = tid; k < p.B * H; k += kConsumers) {
      const int b = k / H;
      float x;
      if (p.h_in) {
        x = p.h_in[k];
      } else {
        int t = p.tokens[b];
        if (t < 0 || t >= p.V) {
          if (k % H == 0 && cta == 0) atomicCAS(p.err, 0, kErrToken);
          t = 0;
        }
        x = __bfloat162float(p.embed[(size_t)t * H + k % H]);
      }
      ha()[k] = x;
    }
    consumer_sync();
  }

  // RMSNorm operand of the tensor-core products: zt rows (2b, 2b + 1) = the
  // hi and lo bf16 terms of gain * x_b, and inv[b] = 1/rms(x_b). Ends on a
  // barrier.
  __device__ __forceinline__ void norm_operand(const float* x, const __nv_bfloat16* gain) {
    const int H = p.H;
    float ss[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) ss[b] = 0.f;
    __nv_bfloat16* z = zt();
    for (int k = tid; k < p.B * H; k += kConsumers) {
      const int b = k / H, e = k % H;
      const float v = x[k];
      __nv_bfloat16 hi, lo;
      split_bf16(v * __bfloat162float(gain[e]), hi, lo);
      z[(size_t)(2 * b) * zt_stride() + e] = hi;
      z[(size_t)(2 * b + 1) * zt_stride() + e] = lo;
#pragma unroll
      for (int bb = 0; bb < NB; ++bb)
        if (bb == b) ss[bb] += v * v;
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const float t = warp_sum(ss[b]);
      if (lane == 0) ssp()[warp * kMaxB + b] = t;
    }
    consumer_sync();
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float t = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < kConsumerWarps; ++w2) t += ssp()[w2 * kMaxB + b];
      inv[b] = rsqrtf(t / (float)H + p.eps);
    }
  }
  __device__ __forceinline__ float inv_of(int b) const {
    float v = inv[0];
#pragma unroll
    for (int bb = 1; bb < NB; ++bb)
      if (bb == b) v = inv[bb];
    return v;
  }

  // All rows of one or two chunks (nr rows of K, phase rows j0 ..; rows
  // [0, cap) at shared address st, the rest at st2 (bf16 only); j0 a multiple
  // of 8, so row r has swizzle r mod 8) on this warp,
  // over the whole K: ys[(j0 + r) * 4 + b] = sum_k W[r][k] x_b[k]. A = 16-row
  // tiles of the chunk (rows past nr read zeros), B = the 2B operand rows at
  // `ob` (column 2b + t = term t of batch row b); loads of 4 k-steps are
  // issued before their products.
  __device__ __forceinline__ void chunk_rows(uint32_t st, uint32_t st2, int cap, int j0, int nr,
                                             int K, uint32_t ob, uint32_t ostride) {
    const int gq = lane >> 2, q = lane & 3, twoB = 2 * p.B;
    const uint32_t zero = zero_addr();
    float* y = ys();
    for (int t0 = 0; t0 < nr; t0 += 16) {
      float d[4][4];
#pragma unroll
      for (int c = 0; c < 4; ++c) d[c][0] = d[c][1] = d[c][2] = d[c][3] = 0.f;
      if constexpr (!Q8) {
        const int row = t0 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const bool arow = row < nr;
        const uint32_t rb = (row < cap ? st + (uint32_t)row * 2u * K
                                       : st2 + (uint32_t)(row - cap) * 2u * K),
                       sw = (uint32_t)(row & 7);
        const int n = lane & 7;
        const bool brow = n < twoB;
        const uint32_t bb = brow ? ob + n * ostride + (((lane >> 3) & 1) << 4) : zero;
        const uint32_t bstep = brow ? 32u : 0u;
        for (int ks = 0; ks < K / 16; ks += 4) {
          uint32_t a[4][4], b[4][2];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t u = (uint32_t)((ks + j) * 2 + (lane >> 4));
            ldsm_x4(arow ? rb + ((u ^ sw) << 4) : zero, a[j]);
            ldsm_x2(bb + (uint32_t)(ks + j) * bstep, b[j]);
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) mma16816(d[j], a[j], b[j]);
        }
      } else {
        // Q8_0: each thread takes 8 consecutive codes of rows gq and gq + 8
        // (columns 32 blk + 8 q ..) and the same 8 operand columns, a column
        // order both operands share; each 32-column block's product is scaled
        // by its rows' scales.
        const int r0 = t0 + gq, r1 = r0 + 8;
        const bool h0 = r0 < nr, h1 = r1 < nr, hb = gq < twoB;
        const uint32_t c0a = st + (uint32_t)r0 * K, c1a = st + (uint32_t)r1 * K;
        const uint32_t sca = st + (uint32_t)nr * K;  // the chunk's scales follow its codes
        const uint32_t s0a = sca + (uint32_t)r0 * (K / 16), s1a = sca + (uint32_t)r1 * (K / 16);
        const int units = K / 16;  // rows r0 and r1 are both gq mod 8
        const uint32_t bbq = ob + gq * ostride + q * 16;
        const uint32_t half = (uint32_t)(q & 1) * 8u;
        for (int blk0 = 0; blk0 < K / 32; blk0 += 2) {  // K / 32 is even
#pragma unroll
        for (int jb = 0; jb < 2; ++jb) {
          const int blk = blk0 + jb;
          const uint32_t u = (uint32_t)swz(blk * 2 + (q >> 1), gq, units);
          const uint2 c0 = h0 ? lds64(c0a + (u << 4) + half) : make_uint2(0u, 0u);
          const uint2 c1 = h1 ? lds64(c1a + (u << 4) + half) : make_uint2(0u, 0u);
          const uint4 z = hb ? lds128(bbq + (uint32_t)blk * 64u) : make_uint4(0u, 0u, 0u, 0u);
          const uint32_t a0[4] = {i8x2_bf16(c0.x, 0), i8x2_bf16(c1.x, 0), i8x2_bf16(c0.x, 1),
                                  i8x2_bf16(c1.x, 1)};
          const uint32_t a1[4] = {i8x2_bf16(c0.y, 0), i8x2_bf16(c1.y, 0), i8x2_bf16(c0.y, 1),
                                  i8x2_bf16(c1.y, 1)};
          const uint32_t b0[2] = {z.x, z.y}, b1[2] = {z.z, z.w};
          float e[4] = {0.f, 0.f, 0.f, 0.f};
          mma16816(e, a0, b0);
          mma16816(e, a1, b1);
          const float sc0 = h0 ? lds_half(s0a + blk * 2) : 0.f;
          const float sc1 = h1 ? lds_half(s1a + blk * 2) : 0.f;
          d[jb][0] = fmaf(sc0, e[0], d[jb][0]);
          d[jb][1] = fmaf(sc0, e[1], d[jb][1]);
          d[jb][2] = fmaf(sc1, e[2], d[jb][2]);
          d[jb][3] = fmaf(sc1, e[3], d[jb][3]);
        }
        }
      }
      // rows gq (d[.][0..1]) and gq + 8 (d[.][2..3]); columns 2q (hi), 2q + 1 (lo)
      const float lo_row = ((d[0][0] + d[1][0]) + (d[2][0] + d[3][0])) +
                           ((d[0][1] + d[1][1]) + (d[2][1] + d[3][1]));
      const float hi_row = ((d[0][2] + d[1][2]) + (d[2][2] + d[3][2])) +
                           ((d[0][3] + d[1][3]) + (d[2][3] + d[3][3]));
      if (q < p.B) {
        if (t0 + gq < nr) y[(j0 + t0 + gq) * 4 + q] = lo_row;
        if (t0 + gq + 8 < nr) y[(j0 + t0 + gq + 8) * 4 + q] = hi_row;
      }
    }
  }

  // The rows of phase `ph` into ys, chunk by chunk: chunk i of the ring goes
  // to warp i mod lm_owners, which waits for it, computes all its rows over
  // the whole K and releases it at once; the other warps only advance their
  // cursor. No CTA barrier until the phase's end, so the products overlap the
  // copies of the next chunks. Ends on a barrier.
  //
  // Chunks of 8 rows go to their owner in pairs (one full 16-row tile); the
  // owners of pairs are at most half a ring of warps, so a warp's owned
  // chunks stay within a ring of each other (the condition under which the
  // owner-mode wait cannot mistake an older phase of a barrier).
  __device__ void rows_product(int ph, uint32_t ob, uint32_t ostride) {
    const int R = p.geo.n[ph], Kp = p.geo.K[ph], cap = cap_rows(Kp, Q8), nch = (R + cap - 1) / cap;
    const int per = (!Q8 && cap < 16) ? 2 : 1;
    const int W = per == 1 ? p.lm_owners : max(1, min(p.lm_owners, r.n / 2));
    for (int c = 0; c < nch; c += per) {
      const int ng = min(per, nch - c);
      if ((int)(grp % (unsigned)W) == warp) {
        const unsigned char* st = chunk_wait_owned(0);
        const unsigned char* st2 = ng > 1 ? chunk_wait_owned(1) : st;
        const int j0 = c * cap;
        if (!warp_quit())
          chunk_rows(su32(st), su32(st2), cap, j0, min(ng * cap, R - j0), Kp, ob, ostride);
        for (int g2 = 0; g2 < ng; ++g2) chunk_release_owned(g2);
      }
      for (int g2 = 0; g2 < ng; ++g2) cursor_advance();
      ++grp;
    }
    consumer_sync();
  }

  __device__ __forceinline__ void tr(int layer, int k) {
    if (p.trace && tid == 0)
      p.trace[((size_t)cta * (p.L + 1) + layer) * kTraceSlots + k] = clock64();
  }
  __device__ __forceinline__ void capture_rows(int slot, const float* x) {
    if (!p.capture || cta != 0) return;
    for (int k = tid; k < p.B * p.H; k += kConsumers) {
      const int b = k / p.H, e = k % p.H;
      p.capture[((size_t)slot * p.capture_stride + b) * p.H + e] = x[k];
    }
  }

  // ---- phase A -------------------------------------------------------------

  // Per-head RMSNorm (+ gain) and rotate-half RoPE of one head held by this
  // warp (d values from `x`), into out[0..d) times `scale`.
  __device__ __forceinline__ void head_norm_rope(const float* x, const __nv_bfloat16* gain,
                                                 int pos, float scale, float* out) {
    const int d = p.d, half = d / 2;
    const float2* rp = p.rope + (size_t)pos * half;
    float ss = 0.f;
    for (int i = lane; i < d; i += 32) ss += x[i] * x[i];
    ss = warp_sum(ss);
    const float iv = rsqrtf(ss / (float)d + p.eps);
    for (int i = lane; i < half; i += 32) {
      const float a = x[i] * iv * __bfloat162float(gain[i]);
      const float c = x[half + i] * iv * __bfloat162float(gain[half + i]);
      const float2 cs = rp[i];
      out[i] = (a * cs.x - c * cs.y) * scale;
      out[half + i] = (c * cs.x + a * cs.y) * scale;
    }
  }

  // q heads (normalised, rotated, scaled by 1/sqrt(d)), k (normalised,
  // rotated, rounded to bf16 as the cache stores it) and v (bf16) of every
  // batch row from the exchanged raw rows; rank 0 appends k and v to the
  // cache. Ends on a barrier.
  __device__ __forceinline__ void prep_heads(int l) {
    const LayerDev& Lw = layer_s(p, l);
    const int d = p.d, rep = p.geo.repc, nroles = rep + 2, rowlen = nroles * d;
    const bool owner = rk == 0 && hs == 0;  // appends the head's k and v
    float* tmp = ssc();  // [11][128] scratch of the k rows
    for (int u = warp; u < p.B * nroles; u += kConsumerWarps) {
      const int b = u / nroles, role = u % nroles, pos = p.pos[b];
      const float* x = raw() + b * rowlen + role * d;
      if (role < rep) {
        head_norm_rope(x, Lw.q_norm, pos, rsqrtf((float)d), qs() + (b * rep + role) * d);
      } else if (role == rep) {
        float* kt = tmp + warp * 128;
        head_norm_rope(x, Lw.k_norm, pos, 1.f, kt);
        __syncwarp();
        const size_t off = kv_off(p, l, b, pos, g);
        for (int i2 = lane; i2 < d; i2 += 32) {
          const __nv_bfloat16 kb = __float2bfloat16_rn(kt[i2]);
          kcur()[b * d + i2] = kb;
          if (owner && !quit) p.kv.k[off + i2] = kb;
        }
      } else {
        const size_t off = kv_off(p, l, b, pos, g);
        for (int i2 = lane; i2 < d; i2 += 32) {
          const __nv_bfloat16 vb = __float2bfloat16_rn(x[i2]);
          vcur()[b * d + i2] = vb;
          if (owner && !quit) p.kv.v[off + i2] = vb;
        }
      }
    }
    consumer_sync();
  }

  __device__ __forceinline__ void phase_a(int l) {
    tr(l, 0);
    const LayerDev& Lw = layer_s(p, l);
    const int d = p.d, rep = p.geo.repc;
    if (l == p.l0)
      first_input();
    else
      exchange_sum(p.pd, tag_of(p.tag0, l - 1, p.l0, 1), hm(), ha());
    tr(l, 1);
    capture_rows(l, ha());
    norm_operand(ha(), Lw.attn_norm);
    const int nA = p.geo.nA, rowlen = (rep + 2) * d, cs = p.geo.cs;
    rows_product(kPA, su32(zt()), (uint32_t)zt_stride() * 2);
    tr(l, 2);
    // the raw q | k | v rows to every CTA of the cluster
    xarm((uint32_t)(p.B * rowlen * 4));
    for (int w = tid; w < nA * p.B * cs; w += kConsumers) {
      const int dest = w / (nA * p.B), v = w % (nA * p.B), j = v / p.B, b = v % p.B;
      xsend(raw() + b * rowlen + rk * nA + j, dest, __float_as_uint(ys()[j * 4 + b] * inv_of(b)));
    }
    xwait();
    prep_heads(l);
    tr(l, 3);
  }

  // ---- phase B -------------------------------------------------------------

  // Run state of the CTA's partial softmax, per query head: m, l, alpha.
  __device__ float* run_m() { return ssc() + 2 * kPage; }
  __device__ float* run_l() { return run_m() + 2; }
  __device__ float* run_a() { return run_m() + 4; }

  // One segment of nk <= 64 keys (rows of d bf16 at Kp / Vp) for batch row b:
  // scores, online-softmax update and P*V into `o` (thread t < rep*d holds
  // output (t / d, t % d)). Ends on a barrier.
  __device__ void attend(int b, const __nv_bfloat16* Kp, const __nv_bfloat16* Vp, int nk,
                         float& o) {
    const int d = p.d, rep = p.geo.repc;
    float* s = ssc();  // [rep][64]
    const float* q = qs() + b * rep * d;
    for (int pr = warp; pr < nk * rep; pr += kConsumerWarps) {
      const int j = pr / rep, h = pr % rep;
      float t = 0.f;
      for (int i = lane; i < d; i += 32)
        t = fmaf(q[h * d + i], __bfloat162float(Kp[(size_t)j * d + i]), t);
      t = warp_sum(t);
      if (lane == 0) s[h * kPage + j] = t;
    }
    consumer_sync();
    if (warp < rep) {
      const int h = warp;
      float mx = -INFINITY;
      for (int j = lane; j < nk; j += 32) mx = fmaxf(mx, s[h * kPage + j]);
      mx = warp_max(mx);
      const float mo = run_m()[h], mn = fmaxf(mo, mx);
      const float alpha = (mo == -INFINITY) ? 0.f : expf(mo - mn);
      float ls = 0.f;
      for (int j = lane; j < nk; j += 32) {
        const float e = expf(s[h * kPage + j] - mn);
        s[h * kPage + j] = e;
        ls += e;
      }
      ls = warp_sum(ls);
      __syncwarp();
      if (lane == 0) {
        run_m()[h] = mn;
        run_l()[h] = run_l()[h] * alpha + ls;
        run_a()[h] = alpha;
      }
    }
    consumer_sync();
    if (tid < rep * d) {
      const int h = tid / d, dim = tid % d;
      float acc = o * run_a()[h];
      for (int j = 0; j < nk; ++j)
        acc = fmaf(s[h * kPage + j], __bfloat162float(Vp[(size_t)j * d + dim]), acc);
      o = acc;
    }
    consumer_sync();
  }

  __device__ __forceinline__ void phase_b(int l) {
    const int H = p.H, d = p.d, rep = p.geo.repc, RD = p.geo.RDc, F = p.geo.F, cs = p.geo.cs;
    xarm((uint32_t)(cs * p.B * (2 + F) * 4));
    for (int b = 0; b < p.B; ++b) {
      if (tid < rep) {
        run_m()[tid] = -INFINITY;
        run_l()[tid] = 0.f;
      }
      consumer_sync();
      float o = 0.f;
      int k0, k1;
      slice(p.pos[b], cs, rk, k0, k1);
      for (int j0 = k0; j0 < k1;) {
        const int je = min(k1, (j0 / kPage + 1) * kPage);
        const __nv_bfloat16* Kp = reinterpret_cast<const __nv_bfloat16*>(chunk_wait(0));
        const __nv_bfloat16* Vp = reinterpret_cast<const __nv_bfloat16*>(chunk_wait(1));
        attend(b, Kp, Vp, je - j0, o);
        chunk_release();
        chunk_release();
        j0 = je;
      }
      if (rk == 0) attend(b, kcur() + b * d, vcur() + b * d, 1, o);  // the new key
      // this CTA's state of each output element to the element's owner
      if (tid < RD) {
        const int h = tid / d, f = tid % F, dest = tid / F;
        float* slot = att() + (rk * kMaxB + b) * (2 + F);
        xsend(slot + 2 + f, dest, __float_as_uint(o));
        if (f == 0) {
          xsend(slot, dest, __float_as_uint(run_m()[h]));
          xsend(slot + 1, dest, __float_as_uint(run_l()[h]));
        }
      }
      consumer_sync();  // run state is reset for the next row
    }
    tr(l, 4);
    xwait();
    // merge the cs states of the F outputs this CTA owns
    if (tid < p.B * F) {
      const int b = tid / F, f = tid % F;
      float M = -INFINITY;
      for (int s2 = 0; s2 < cs; ++s2) M = fmaxf(M, att()[(s2 * kMaxB + b) * (2 + F)]);
      float Ls = 0.f, Os = 0.f;
      for (int s2 = 0; s2 < cs; ++s2) {
        const float* e = att() + (s2 * kMaxB + b) * (2 + F);
        const float w = (e[0] == -INFINITY) ? 0.f : expf(e[0] - M);
        Ls = fmaf(e[1], w, Ls);
        Os = fmaf(e[2 + f], w, Os);
      }
      cmb()[b * F + f] = Os / Ls;
    }
    consumer_sync();
    // the merged outputs (hi and lo bf16 terms, pairs of columns) to every CTA
    xarm((uint32_t)(p.B * RD * 2 * 2));
    const int F2 = F / 2;
    for (int w = tid; w < p.B * F2 * cs; w += kConsumers) {
      const int dest = w / (p.B * F2), v = w % (p.B * F2), b = v / F2, f = 2 * (v % F2);
      __nv_bfloat16 h0, l0, h1, l1;
      split_bf16(cmb()[b * F + f], h0, l0);
      split_bf16(cmb()[b * F + f + 1], h1, l1);
      const int col = rk * F + f;
      xsend(zo() + (size_t)(2 * b) * zo_stride() + col, dest, pack2(h0, h1));
      xsend(zo() + (size_t)(2 * b + 1) * zo_stride() + col, dest, pack2(l0, l1));
    }
    xwait();
    tr(l, 5);
    // O projection rows of this CTA
    const int nO = p.geo.nO;
    rows_product(kPO, su32(zo()), (uint32_t)zo_stride() * 2);
    const uint32_t tag = tag_of(p.tag0, l, p.l0, 0);
    if (l != p.withhold_layer && !quit)
      for (int t = tid; t < nO * p.B; t += kConsumers) {
        const int j = t / p.B, b = t % p.B;
        st_tag(p.po + ((size_t)cl * kMaxB + b) * H + rk * nO + j, ys()[j * 4 + b], tag);
      }
    tr(l, 6);
  }

  // ---- phase C -------------------------------------------------------------

  __device__ __forceinline__ void phase_c(int l) {
    const LayerDev& Lw = layer_s(p, l);
    const int H = p.H, nc = p.geo.nc, Kc = p.geo.Kc, cs = p.geo.cs;
    exchange_sum(p.po, tag_of(p.tag0, l, p.l0, 0), ha(), hm());
    tr(l, 7);
    norm_operand(hm(), Lw.ffn_norm);
    rows_product(kPGU, su32(zt()), (uint32_t)zt_stride() * 2);
    for (int t = tid; t < nc * p.B; t += kConsumers) {
      const int j = t / p.B, b = t % p.B;
      const float y = ys()[j * 4 + b] * inv_of(b), z = ys()[(nc + j) * 4 + b] * inv_of(b);
      act()[b * nc + j] = y / (1.f + expf(-y)) * z;
    }
    consumer_sync();
    tr(l, 8);
    xarm((uint32_t)(p.B * Kc * 2 * 2));
    const int n2 = nc / 2;
    for (int w = tid; w < p.B * n2 * cs; w += kConsumers) {
      const int dest = w / (p.B * n2), v = w % (p.B * n2), b = v / n2, j = 2 * (v % n2);
      __nv_bfloat16 h0, l0, h1, l1;
      split_bf16(act()[b * nc + j], h0, l0);
      split_bf16(act()[b * nc + j + 1], h1, l1);
      const int col = rk * nc + j;
      xsend(za() + (size_t)(2 * b) * za_stride() + col, dest, pack2(h0, h1));
      xsend(za() + (size_t)(2 * b + 1) * za_stride() + col, dest, pack2(l0, l1));
    }
    xwait();
    tr(l, 9);
    const int nO = p.geo.nO;
    rows_product(kPD, su32(za()), (uint32_t)za_stride() * 2);
    const uint32_t tag = tag_of(p.tag0, l, p.l0, 1);
    if (!quit)
      for (int t = tid; t < nO * p.B; t += kConsumers) {
        const int j = t / p.B, b = t % p.B;
        st_tag(p.pd + ((size_t)cl * kMaxB + b) * H + rk * nO + j, ys()[j * 4 + b], tag);
      }
    tr(l, 10);
  }

  // ---- tail: final norm + LM head + greedy ---------------------------------

  __device__ __forceinline__ void fold_logit(int bb, int id, float y) {
    if (p.logits) p.logits[(size_t)bb * p.V + id] = y;
    if (isfinite(y)) {
      const uint32_t uu = (y == 0.f) ? 0u : __float_as_uint(y);  // -0 ranks as +0
      const uint32_t ord = (uu & 0x80000000u) ? ~uu : (uu | 0x80000000u);
      const unsigned long long key = ((unsigned long long)ord << 32) | (0xffffffffu - (uint32_t)id);
#pragma unroll
      for (int b2 = 0; b2 < kMaxB; ++b2)
        if (b2 == bb && key > wbest[b2]) wbest[b2] = key;
    }
  }
  // One LM-head chunk (nr <= 8 whole embedding rows, contiguous) on this
  // warp: logits of every batch row, folded into the greedy keys. Each
  // thread loads 8 consecutive columns (32 blk + 8 q ..) of row gq and of
  // operand row gq, a column order both operands share; rows 8..15 of the
  // tile are zero.
  __device__ __forceinline__ void lm_rows(const unsigned char* st, int n0, int nr) {
    const int gq = lane >> 2, q = lane & 3, H = p.H;
    const bool ha = gq < nr, hb = gq < 2 * p.B;
    const uint32_t ab = su32(st) + gq * 2 * H + q * 16;
    const uint32_t bb = su32(zt()) + gq * zt_stride() * 2 + q * 16;
    float d0[4] = {0.f, 0.f, 0.f, 0.f}, d1[4] = {0.f, 0.f, 0.f, 0.f};
    for (int blk = 0; blk < H / 32; ++blk) {
      const uint4 w = ha ? lds128(ab + blk * 64) : make_uint4(0u, 0u, 0u, 0u);
      const uint4 z = hb ? lds128(bb + blk * 64) : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t a0[4] = {w.x, 0u, w.y, 0u}, a1[4] = {w.z, 0u, w.w, 0u};
      const uint32_t b0[2] = {z.x, z.y}, b1[2] = {z.z, z.w};
      mma16816(d0, a0, b0);
      mma16816(d1, a1, b1);
    }
    if (ha && q < p.B) fold_logit(q, n0 + gq, ((d0[0] + d1[0]) + (d0[1] + d1[1])) * inv_of(q));
  }

  __device__ __forceinline__ void finish_head() {
    unsigned long long* bst = best();
    if (tid < kMaxB) bst[tid] = 0ull;
    consumer_sync();
#pragma unroll
    for (int bb = 0; bb < kMaxB; ++bb) {
      unsigned long long k = wbest[bb];
      for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long other = __shfl_xor_sync(0xffffffffu, k, o);
        k = other > k ? other : k;
      }
      if (lane == 0 && bb < p.B && k) atomicMax(bst + bb, k);
    }
    consumer_sync();
    if (tid < p.B && !quit && bst[tid]) atomicMax(p.am_key + tid, bst[tid]);
    __threadfence();
    consumer_sync();
    if (tid == 0) {
      const unsigned int old = atomicAdd(p.am_cnt, 1u);
      *flag() = (old == (unsigned int)G - 1);
    }
    consumer_sync();
    if (*flag()) {
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
  }

  __device__ __forceinline__ void tail() {
    const int L = p.L;
    tr(L, 0);
    exchange_sum(p.pd, tag_of(p.tag0, p.l1 - 1, p.l0, 1), hm(), ha());
    tr(L, 1);
    capture_rows(p.l1, ha());
    if (cta == 0 && p.h_out)
      for (int k = tid; k < p.B * p.H; k += kConsumers) p.h_out[k] = ha()[k];
    if (!p.run_head) return;
    norm_operand(ha(), p.final_norm);
    int a, b;
    slice(p.V, G, cta, a, b);
    const int cap = p.lm_rows;
    for (int n = a; n < b;) {
      const int e = min(b, n + cap), nr = e - n;
      if ((int)(i % p.lm_owners) == warp) {
        const unsigned char* st = chunk_wait_owned();
        if (!warp_quit()) lm_rows(st, n, nr);
        __syncwarp();
        if (lane == 0 && !quit) mbar_arrive_n(&r.empty[stage], kConsumerWarps);
      }
      cursor_advance();
      n = e;
    }
    tr(L, 2);
    finish_head();
    tr(L, 4);
  }
};

template <int NB, bool Q8>
__global__ void __launch_bounds__(kThreads, 1) decode_cluster_kernel(const __grid_constant__ Params p) {
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
  uint64_t* xbar = ring.empty + kMaxStages;
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.n_stages; ++s) {
      mbar_init(&ring.full[s], 1);
      mbar_init(&ring.empty[s], kConsumerWarps);
    }
    mbar_init(&xbar[0], 1);
    mbar_init(&xbar[1], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
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
    if (threadIdx.x < 16)  // zero bytes read by the tensor-core loads of padding rows
      reinterpret_cast<uint32_t*>(smem + p.off_misc)[threadIdx.x] = 0u;
  }
  // every CTA's barriers are initialised before any peer may signal them
  cluster_sync_all();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, c = blockIdx.x;
  unsigned long long* trow =
      p.trace ? p.trace + ((size_t)c * (p.L + 1) + p.L) * kTraceSlots : nullptr;
  if (trow && threadIdx.x == 0) {
    trow[12] = now_ns();
    trow[13] = clock64();
  }
  volatile unsigned int* counts = reinterpret_cast<volatile unsigned int*>(smem + p.off_misc + 104);
  bool quit_any = false;
  if (warp == kConsumerWarps) {
    if (lane == 0) {
      Producer pr(*ps, ring);
      const int cl = c / p.geo.cs, rk = (int)cluster_rank();
      for (int l = p.l0; l < p.l1 && !pr.quit; ++l) pr.layer(l, cl, cl / p.geo.split, rk);
      int a, b;
      slice(p.V, gridDim.x, c, a, b);
      if (!pr.quit) pr.tail(a, b);
      if (trow) trow[3] = clock64();
      counts[0] = pr.i;
    }
  } else {
    Consumer<NB, Q8> cs(*ps, ring, smem);
    // `quit` is per thread, so it steers no path that holds a barrier: after
    // an abort every thread still walks all phases (waits return at once, no
    // global stores), and every exchange still sends its bytes.
    for (int l = p.l0; l < p.l1; ++l) {
      cs.cur_layer = l;
      cs.phase_a(l);
      cs.phase_b(l);
      cs.phase_c(l);
    }
    cs.tail();
    quit_any = consumer_sync_or(cs.quit);
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
    const unsigned int issued = counts[0], n = (unsigned int)ring.n;
    const unsigned int first = issued > n ? issued - n : 0u;
    for (unsigned int k = first; k < issued; ++k) {
      const unsigned long long t0 = now_ns();
      while (!mbar_test(&ring.full[k % n], (k / n) & 1))
        if (now_ns() - t0 > 10000000ull) break;  // 10 ms
    }
  }
  // No CTA leaves while a peer may still store into its shared memory: every
  // peer has issued all its exchanges once this barrier completes; after an
  // abort, stores issued just before it are given time to land.
  cluster_sync_all();
  if (quit_any && threadIdx.x == 0) {
    const unsigned long long t0 = now_ns();
    while (now_ns() - t0 < 50000ull) {
    }
  }
  cluster_sync_all();
}

// Packs one block's weights into the per-CTA images: block (cta, row j,
// phase) copies row j of the CTA's rows of that phase (bf16 elements, or
// Q8_0 codes then scales), its 16-byte units at u ^ (j mod 8).
struct PackArgs {
  const void* w[kNumLin];
  const __half* s[kNumLin];
  int H, nq, nkv, d, I;
  Geo geo;
  int q8;
  unsigned char* dst;  // this block's images: [clusters][cs][stream_bytes]
  int stream_bytes;
  int pofs[4];
};

__global__ void pack_kernel(const PackArgs a) {
  const Geo& G = a.geo;
  const int cta = blockIdx.x, j = blockIdx.y, ph = blockIdx.z;
  const int* n = G.n;
  if (j >= n[ph]) return;
  const bool q8 = a.q8 != 0;
  const int cl = cta / G.cs, r = cta % G.cs, g = cl / G.split, hs = cl % G.split;
  const int Kp = G.K[ph], RD = G.RDc;
  const int q0 = (g * (a.nq / a.nkv) + hs * G.repc) * a.d;  // first q row / Wo column of the cluster
  int lin, kfull, col0;
  size_t row;
  if (ph == kPA) {
    const int rho = r * n[kPA] + j;
    kfull = a.H;
    col0 = 0;
    if (rho < RD) {
      lin = kWq;
      row = (size_t)q0 + rho;
    } else if (rho < RD + a.d) {
      lin = kWk;
      row = (size_t)g * a.d + rho - RD;
    } else {
      lin = kWv;
      row = (size_t)g * a.d + rho - RD - a.d;
    }
  } else if (ph == kPO) {
    lin = kWo;
    row = (size_t)r * n[kPO] + j;
    kfull = a.nq * a.d;
    col0 = q0;
  } else if (ph == kPGU) {
    const int nc = G.nc, c0 = cl * G.Kc + r * nc;
    lin = j < nc ? kWg : kWu;
    row = (size_t)c0 + (j < nc ? j : j - nc);
    kfull = a.H;
    col0 = 0;
  } else {
    lin = kWd;
    row = (size_t)r * n[kPD] + j;
    kfull = a.I;
    col0 = cl * G.Kc;
  }
  const int cap = cap_rows(Kp, q8), c = j / cap, slot = j - c * cap;
  const int nr = min(cap, n[ph] - c * cap);
  unsigned char* chunk = a.dst + (size_t)cta * a.stream_bytes + a.pofs[ph] +
                         (size_t)c * chunk_bytes(cap, Kp, q8);
  if (!q8) {
    const unsigned short* src =
        static_cast<const unsigned short*>(a.w[lin]) + row * kfull + col0;
    unsigned short* dst = reinterpret_cast<unsigned short*>(chunk + (size_t)slot * 2 * Kp);
    for (int e = threadIdx.x; e < Kp; e += blockDim.x)
      dst[(swz(e >> 3, j, Kp / 8) << 3) | (e & 7)] = src[e];
  } else {
    const unsigned char* src = static_cast<const unsigned char*>(a.w[lin]) + row * kfull + col0;
    unsigned char* dst = chunk + (size_t)slot * Kp;
    for (int e = threadIdx.x; e < Kp; e += blockDim.x)
      dst[(swz(e >> 4, j, Kp / 16) << 4) | (e & 15)] = src[e];
    const __half* ssrc = a.s[lin] + row * (kfull / 32) + col0 / 32;
    __half* sdst = reinterpret_cast<__half*>(chunk + (size_t)nr * Kp + (size_t)slot * (Kp / 16));
    for (int t = threadIdx.x; t < Kp / 32; t += blockDim.x) sdst[t] = ssrc[t];
  }
}

}  // namespace clus

// ---------------------------------------------------------------------------
// Host side

namespace {

struct ClusterState {
  unsigned long long* po = nullptr;
  unsigned long long* pd = nullptr;
  unsigned long long* am_key = nullptr;
  unsigned int* am_cnt = nullptr;
  int* abort_flag = nullptr;
  LayerDev* layers = nullptr;
  unsigned char* packed = nullptr;
  int stream_bytes = 0;
  int pofs[4] = {0, 0, 0, 0};
  clus::Geo geo{};
  uint32_t next_tag = 1;
  bool eligible = false;
  unsigned long long wait_ns = 1000000000ull;
  int withhold = -1;
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// The split (cs CTAs per cluster, split clusters per kv head) covers the
// shape: every per-CTA share is whole and fits the kernel's buffers.
bool geo_ok(const Shape& s, const clus::Geo& g) {
  if (g.cs > clus::kMaxCS || s.nkv < 1 || s.nq % s.nkv || (s.nq / s.nkv) % g.split) return false;
  if (s.H > clus::kMaxH || s.H % 64 || s.d % 64 || s.d > 128) return false;
  if ((g.repc + 2) * s.d % g.cs || g.nA > clus::kMaxRows || g.nA < 1) return false;
  if (g.RDc % 64 || g.RDc > 256 || g.RDc % g.cs || g.F % 2 || s.d % g.F) return false;
  if (s.H % g.cs || g.nO > clus::kMaxRows) return false;
  if (s.I % (g.ncl * g.cs) || g.nc < 1 || g.nc % 2 || 2 * g.nc > clus::kMaxRows) return false;
  if (g.Kc % 64) return false;
  if (s.L > 64 || s.V >= 0x7fffffff) return false;
  return true;
}

void state_free(ClusterState* st) {
  void* bufs[] = {st->po, st->pd, st->am_key, st->am_cnt, st->abort_flag, st->layers, st->packed};
  for (void* b : bufs)
    if (b) cudaFree(b);
}

const void* kernel_for(int B, bool q8) {
  if (q8)
    return B == 1 ? (const void*)clus::decode_cluster_kernel<1, true>
                  : (const void*)clus::decode_cluster_kernel<4, true>;
  return B == 1 ? (const void*)clus::decode_cluster_kernel<1, false>
                : (const void*)clus::decode_cluster_kernel<4, false>;
}

}  // namespace

fs_status cluster_init(fs_model* m) {
  ClusterState* st = new ClusterState();
  m->cl_extras = st;
  const Shape& s = m->s;
  // The first split whose clusters all fit on the device at once: 16-CTA
  // clusters, one per kv head; 8-CTA clusters, two per kv head; 8-CTA
  // clusters, one per kv head.
  st->eligible = false;
  const int splits[3][2] = {{16, 1}, {8, 2}, {8, 1}};
  for (const auto& sp : splits) {
    const int cs = sp[0];
    const clus::Geo g = clus::make_geo(s.H, s.nq, s.nkv, s.d, s.I, cs, sp[1]);
    if (!geo_ok(s, g)) continue;
    bool fits = true;
    for (int nb : {1, 4}) {
      const void* k = kernel_for(nb, m->q8);
      if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448) !=
              cudaSuccess ||
          cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
              cudaSuccess) {
        cudaGetLastError();
        fits = false;
        break;
      }
      cudaLaunchConfig_t cfg{};
      cfg.gridDim = dim3(g.ncl * cs);
      cfg.blockDim = dim3(clus::kThreads);
      cfg.dynamicSmemBytes = 232448;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = cs;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, k, &cfg) != cudaSuccess || n < g.ncl) {
        cudaGetLastError();
        fits = false;
        break;
      }
    }
    if (fits) {
      st->geo = g;
      st->eligible = true;
      break;
    }
  }
  if (!st->eligible) return FS_OK;
  const clus::Geo& G = st->geo;
  auto alloc = [&](void** p, size_t bytes) {
    if (cudaMalloc(p, bytes) != cudaSuccess) {
      cudaGetLastError();
      *p = nullptr;
      return false;
    }
    cudaMemset(*p, 0, bytes);
    return true;
  };
  int acc = 0;
  for (int ph = 0; ph < clus::kPhases; ++ph) {
    st->pofs[ph] = acc;
    acc += clus::phase_bytes(G.n[ph], G.K[ph], m->q8);
  }
  st->stream_bytes = acc;
  const size_t image = (size_t)G.ncl * G.cs * acc;  // one block's images
  const size_t words = (size_t)G.ncl * clus::kMaxB * s.H * sizeof(unsigned long long);
  bool ok = alloc((void**)&st->po, words) && alloc((void**)&st->pd, words) &&
            alloc((void**)&st->am_key, clus::kMaxB * sizeof(unsigned long long)) &&
            alloc((void**)&st->am_cnt, 64) && alloc((void**)&st->abort_flag, 64) &&
            alloc((void**)&st->layers, (size_t)s.L * sizeof(LayerDev)) &&
            alloc((void**)&st->packed, image * s.L);
  if (ok) {
    for (int l = 0; l < s.L; ++l) {
      clus::PackArgs a{};
      for (int t = 0; t < kNumLin; ++t) {
        a.w[t] = m->layers[l].w[t];
        a.s[t] = m->layers[l].s[t];
      }
      a.H = s.H; a.nq = s.nq; a.nkv = s.nkv; a.d = s.d; a.I = s.I;
      a.geo = G;
      a.q8 = m->q8 ? 1 : 0;
      a.dst = st->packed + image * l;
      a.stream_bytes = acc;
      for (int ph = 0; ph < 4; ++ph) a.pofs[ph] = st->pofs[ph];
      clus::pack_kernel<<<dim3(G.ncl * G.cs, clus::kMaxRows, clus::kPhases), 128>>>(a);
    }
    ok = cudaDeviceSynchronize() == cudaSuccess;
    if (!ok) cudaGetLastError();
  }
  if (!ok) {
    state_free(st);
    delete st;
    m->cl_extras = nullptr;
    set_error("out of device memory for the cluster decode kernel's buffers");
    return FS_ERR_OOM;
  }
  cudaMemcpy(st->layers, m->layers.data(), (size_t)s.L * sizeof(LayerDev), cudaMemcpyHostToDevice);
  return FS_OK;
}

void cluster_release(fs_model* m) {
  ClusterState* st = static_cast<ClusterState*>(m->cl_extras);
  if (!st) return;
  state_free(st);
  delete st;
  m->cl_extras = nullptr;
}

void cluster_reset(fs_model* m) {
  ClusterState* st = static_cast<ClusterState*>(m->cl_extras);
  if (!st || !st->eligible) return;
  cudaDeviceSynchronize();
  cudaMemset(st->am_key, 0, clus::kMaxB * sizeof(unsigned long long));
  cudaMemset(st->am_cnt, 0, 64);
  cudaMemset(st->abort_flag, 0, 64);
  st->next_tag += 1u << 20;  // every tag in flight is now stale
}

void cluster_debug_wait(fs_model* m, unsigned long long wait_ns, int withhold_layer) {
  ClusterState* st = static_cast<ClusterState*>(m->cl_extras);
  if (!st) return;
  st->wait_ns = wait_ns;
  st->withhold = withhold_layer;
}

bool cluster_eligible(const fs_model* m) {
  const ClusterState* st = static_cast<const ClusterState*>(m->cl_extras);
  return st && st->eligible;
}

fs_status decode_cluster(fs_model* m, const fs_kv* kv, const RowMap& map, int B,
                         const int32_t* tok, const float* h_in, float* h_out, int l0, int l1,
                         bool run_head, float* logits, int32_t* argmax, cudaStream_t stream) {
  ClusterState* st = static_cast<ClusterState*>(m->cl_extras);
  if (!st || !st->eligible || B > clus::kMaxB || B < 1) return FS_ERR_UNSUPPORTED;
  const Shape& s = m->s;
  clus::Params p{};
  const clus::Geo& G = st->geo;
  p.L = s.L; p.H = s.H; p.nq = s.nq; p.nkv = s.nkv; p.d = s.d; p.I = s.I; p.V = s.V;
  p.geo = G;
  p.eps = s.eps;
  p.layers = st->layers;
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
  p.po = st->po;
  p.pd = st->pd;
  p.q8 = m->q8 ? 1 : 0;
  p.packed = st->packed;
  p.stream_bytes = st->stream_bytes;
  for (int ph = 0; ph < 4; ++ph) p.pofs[ph] = st->pofs[ph];
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
    const size_t words = (size_t)G.ncl * clus::kMaxB * s.H * sizeof(unsigned long long);
    cudaMemsetAsync(st->po, 0, words, stream);
    cudaMemsetAsync(st->pd, 0, words, stream);
    st->next_tag = 1;
  }
  p.tag0 = st->next_tag;
  st->next_tag += 2u * (uint32_t)(l1 - l0) + 1u;
  // shared memory carve-up
  const int rep = G.repc, RD = G.RDc, F = G.F, nc = G.nc, Kc = G.Kc;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes, 128);
    return (int)o;
  };
  int n_items = 0;  // tensor-core work items of the largest product
  for (int ph = 0; ph < clus::kPhases; ++ph)
    n_items = std::max(n_items, (G.n[ph] + 15) / 16 * (G.K[ph] / 64));
  const size_t red = std::max((size_t)n_items * 64 * 4,
                              ((size_t)G.ncl + 1) * B * (s.H / G.cs) * 4);
  const size_t tab_ptrs = (size_t)s.L * sizeof(LayerDev);
  const size_t bt_bytes = (size_t)B * kv->pages_per_seq * sizeof(int32_t);
  const bool bt_smem = bt_bytes <= 8192;
  size_t fixed = 0;
  {
    // first pass: sizes only
    off = 0;
    take((size_t)B * s.H * 4);                      // ha
    take((size_t)B * s.H * 4);                      // hm
    take((size_t)2 * B * (s.H + 8) * 2);            // zt
    take((size_t)2 * B * (RD + 8) * 2);             // zo
    take((size_t)2 * B * (Kc + 8) * 2);             // za
    take((size_t)B * (rep + 2) * s.d * 4);          // raw
    take((size_t)B * RD * 4);                       // q
    take((size_t)2 * clus::kMaxB * s.d * 2);        // kcur, vcur
    take((size_t)G.cs * clus::kMaxB * (2 + F) * 4);  // att
    take((size_t)B * F * 4);                        // cmb
    take((size_t)B * nc * 4);                       // act
    take((size_t)std::max(2 * kPage + 8, clus::kConsumerWarps * 128) * 4);  // ssc
    take((size_t)clus::kMaxRows * 4 * 4);           // ys
    take(red);
    take((size_t)clus::kConsumerWarps * clus::kMaxB * 4);  // ss
    take(1152);                                     // misc
    take((size_t)(2 * clus::kMaxStages + 2) * 8);   // barriers
    take(tab_ptrs + (bt_smem ? bt_bytes : 0));      // tables
    take(sizeof(clus::Params));                     // parameter copy
    fixed = off;
  }
  const size_t budget = 232448;
  int n_stages = (int)((budget - std::min(fixed, budget)) / clus::kStage);
  n_stages = std::min(n_stages, clus::kMaxStages);
  // the most chunks one phase holds at once
  // products take their chunks in passes of at most a ring; an attention
  // segment holds 2 chunks
  if (n_stages < 4) return FS_ERR_UNSUPPORTED;
  off = (size_t)n_stages * clus::kStage;
  p.off_ha = take((size_t)B * s.H * 4);
  p.off_hm = take((size_t)B * s.H * 4);
  p.off_zt = take((size_t)2 * B * (s.H + 8) * 2);
  p.off_zo = take((size_t)2 * B * (RD + 8) * 2);
  p.off_za = take((size_t)2 * B * (Kc + 8) * 2);
  p.off_raw = take((size_t)B * (rep + 2) * s.d * 4);
  p.off_q = take((size_t)B * RD * 4);
  p.off_kv = take((size_t)2 * clus::kMaxB * s.d * 2);
  p.off_att = take((size_t)G.cs * clus::kMaxB * (2 + F) * 4);
  p.off_cmb = take((size_t)B * F * 4);
  p.off_act = take((size_t)B * nc * 4);
  p.off_ssc = take((size_t)std::max(2 * kPage + 8, clus::kConsumerWarps * 128) * 4);
  p.off_ys = take((size_t)clus::kMaxRows * 4 * 4);
  p.off_red = take(red);
  p.off_ss = take((size_t)clus::kConsumerWarps * clus::kMaxB * 4);
  p.off_misc = take(1152);
  p.off_bar = take((size_t)(2 * clus::kMaxStages + 2) * 8);
  p.off_tab = take(tab_ptrs + (bt_smem ? bt_bytes : 0));
  p.off_par = take(sizeof(clus::Params));
  if (off > budget) return FS_ERR_UNSUPPORTED;
  p.bt_in_smem = bt_smem ? 1 : 0;
  p.n_stages = n_stages;
  p.lm_owners = std::min(clus::kConsumerWarps, n_stages);
  p.lm_rows = std::min(8, clus::kStage / (2 * s.H));
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(G.ncl * G.cs);
  cfg.blockDim = dim3(clus::kThreads);
  cfg.dynamicSmemBytes = off;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = G.cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launches();
  cudaError_t e;
  if (m->q8)
    e = B == 1 ? cudaLaunchKernelEx(&cfg, clus::decode_cluster_kernel<1, true>, p)
               : cudaLaunchKernelEx(&cfg, clus::decode_cluster_kernel<4, true>, p);
  else
    e = B == 1 ? cudaLaunchKernelEx(&cfg, clus::decode_cluster_kernel<1, false>, p)
               : cudaLaunchKernelEx(&cfg, clus::decode_cluster_kernel<4, false>, p);
  if (e != cudaSuccess) {
    set_error(std::string("cluster decode kernel launch failed: ") + cudaGetErrorString(e));
    return FS_ERR_CUDA;
  }
  return FS_OK;
}

}  // namespace fs
