// Seeded sampling of one token per row of fp32 logits: temperature, then
// top-k, then top-p over the survivors, renormalise, and an inverse-CDF draw
// in id order with a Philox4x32-10 uniform.
//
// One thread-block cluster of `nr` CTAs per row. CTA r keeps the
// order-preserving keys of ids [r*chunk, (r+1)*chunk) in shared memory, so
// every pass after the first reads shared memory only; cluster-wide sums and
// histograms go through distributed shared memory.
//
// Ranking: logit descending, ties to the lowest id. A threshold is found by
// radix selection on the 32-bit key, 8 bits at a time, MSB first: top-k on
// counts, top-p on probability mass. Masses are fixed-point integers
// (exp((l - max)/T) in units of 2^-32, each at most 2^32), so every sum, and
// with it every decision, is exact and independent of the order of additions.
#include <cooperative_groups.h>

#include "fs_internal.h"

namespace cg = cooperative_groups;

namespace fs {
namespace samp {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr unsigned kNone = 0xffffffffu;

struct Args {
  const float* logits;
  int V, chunk;
  float inv_t;
  int top_k;
  float top_p;
  unsigned long long seed, step;
  int32_t* out;
};

__device__ __forceinline__ uint32_t ord_key(float x) {
  const uint32_t u = __float_as_uint(x == 0.f ? 0.f : x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Philox4x32 with 10 rounds (Salmon et al., SC'11) on counter c, key k; the
// first output word.
__device__ __forceinline__ uint32_t philox_first(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                                 uint32_t k0, uint32_t k1) {
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t lo0 = 0xD2511F53u * c0, hi0 = __umulhi(0xD2511F53u, c0);
    const uint32_t lo1 = 0xCD9E8D57u * c2, hi1 = __umulhi(0xCD9E8D57u, c2);
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  return c0;
}

struct Smem {
  unsigned long long hist[2][256];  // counts or masses of one radix pass
  unsigned long long tot[256];
  unsigned long long warp_part[kWarps];
  unsigned long long slot[16];      // per-CTA values read by the other CTAs of the cluster
  unsigned long long bcast[4];
  float fred[kWarps];
  uint32_t keys[1];                 // [chunk] (dynamic tail)
};

template <typename T>
__device__ __forceinline__ T warp_incl_scan(T v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const T n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// Exclusive prefix of v over the CTA's threads (in thread order); *total = sum.
__device__ unsigned long long block_excl_scan(unsigned long long v, Smem& sm,
                                              unsigned long long* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned long long inc = warp_incl_scan(v, lane);
  if (lane == 31) sm.warp_part[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const unsigned long long w = sm.warp_part[lane];
    const unsigned long long wi = warp_incl_scan(w, lane);
    sm.warp_part[lane] = wi - w;  // exclusive
    if (lane == 31) sm.bcast[0] = wi;
  }
  __syncthreads();
  const unsigned long long r = sm.warp_part[warp] + inc - v;
  *total = sm.bcast[0];
  __syncthreads();
  return r;
}

__device__ unsigned long long block_sum(unsigned long long v, Smem& sm) {
  unsigned long long t;
  block_excl_scan(v, sm, &t);
  return t;
}

// Cluster-wide exclusive prefix (over CTA ranks) and total of a per-CTA value,
// through slot `s` of every CTA.
__device__ void cluster_prefix(cg::cluster_group& cl, Smem& sm, int s, unsigned long long v,
                               unsigned long long* before, unsigned long long* total) {
  if (threadIdx.x == 0) sm.slot[s] = v;
  cl.sync();
  const int nr = (int)cl.num_blocks(), me = (int)cl.block_rank();
  unsigned long long b = 0, t = 0;
  for (int r = 0; r < nr; ++r) {
    const unsigned long long x = *cl.map_shared_rank(&sm.slot[s], r);
    if (r < me) b += x;
    t += x;
  }
  *before = b;
  *total = t;
}

// One radix-select step: the histogram buffer `buf` holds this CTA's bins;
// sums them over the cluster and finds, from the top bin down, the first bin
// at which the running total (starting from `above`) reaches `need`. Returns
// the bin and sets *above to the total of the bins above it.
__device__ int radix_pick(cg::cluster_group& cl, Smem& sm, int buf, unsigned long long need,
                          unsigned long long* above) {
  cl.sync();
  const int nr = (int)cl.num_blocks();
  if (threadIdx.x < 256) {
    unsigned long long t = 0;
    for (int r = 0; r < nr; ++r) t += cl.map_shared_rank(&sm.hist[buf][0], r)[threadIdx.x];
    sm.tot[threadIdx.x] = t;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    // lane l holds bins 255-8l .. 248-8l (descending)
    unsigned long long loc = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) loc += sm.tot[255 - 8 * lane - j];
    const unsigned long long inc = warp_incl_scan(loc, lane);
    const unsigned long long base = *above;
    const bool hit = base + inc >= need;
    const unsigned hits = __ballot_sync(0xffffffffu, hit);
    if (hits) {
      const int l = __ffs(hits) - 1;
      if (lane == l) {
        unsigned long long c = base + inc - loc;
        int b = 255 - 8 * l;
        for (int j = 0; j < 8; ++j, --b) {
          if (c + sm.tot[b] >= need) break;
          c += sm.tot[b];
        }
        if (b < 248 - 8 * l) b = 248 - 8 * l;  // not reached: need <= c + bins
        sm.bcast[1] = (unsigned long long)b;
        sm.bcast[2] = c;
      }
    } else if (lane == 0) {
      // rounding: the need is never reached; take the lowest non-empty bin
      int b = 0;
      while (b < 255 && sm.tot[b] == 0) ++b;
      unsigned long long c = base;
      for (int j = 255; j > b; --j) c += sm.tot[j];
      sm.bcast[1] = (unsigned long long)b;
      sm.bcast[2] = c;
    }
  }
  __syncthreads();
  const int pick = (int)sm.bcast[1];
  *above = sm.bcast[2];
  __syncthreads();
  return pick;
}

__global__ void __launch_bounds__(kThreads, 1) sample_kernel(Args a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  cg::cluster_group cl = cg::this_cluster();
  const int nr = (int)cl.num_blocks(), rank = (int)cl.block_rank();
  const int row = blockIdx.x / nr;
  const int i0 = rank * a.chunk;
  const int n = max(0, min(a.V, i0 + a.chunk) - i0);
  const float* lg = a.logits + (size_t)row * a.V + i0;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // 1. keys and the largest finite logit
  float mx = -INFINITY;
  unsigned long long nfin = 0;
  for (int i = tid; i < n; i += kThreads) {
    const float x = lg[i];
    const bool fin = isfinite(x);
    sm.keys[i] = fin ? ord_key(x) : 0u;
    if (fin) {
      mx = fmaxf(mx, x);
      ++nfin;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) sm.fred[warp] = mx;
  __syncthreads();
  if (tid == 0) {
    float m = -INFINITY;
    for (int w = 0; w < kWarps; ++w) m = fmaxf(m, sm.fred[w]);
    sm.slot[0] = (unsigned long long)ord_key(m == -INFINITY ? -3.0e38f : m);
  }
  const unsigned long long cnt = block_sum(nfin, sm);
  if (tid == 0) sm.slot[1] = cnt;
  cl.sync();
  uint32_t mkey = 0;
  unsigned long long total_fin = 0;
  for (int r = 0; r < nr; ++r) {
    mkey = max(mkey, (uint32_t)*cl.map_shared_rank(&sm.slot[0], r));
    total_fin += *cl.map_shared_rank(&sm.slot[1], r);
  }
  const float m = key_value(mkey);
  if (total_fin == 0) {
    if (tid == 0 && rank == 0) a.out[row] = 0;
    cl.sync();
    return;
  }

  // contiguous per-thread ranges of the CTA's ids (for passes in id order)
  const int cc = (n + kThreads - 1) / kThreads;
  const int r0 = min(n, tid * cc), r1 = min(n, r0 + cc);

  // 2. top-k: threshold key tk; ties at tk kept up to local index cut_k
  uint32_t tk = 0;
  long long cut_k = -1;  // global id of the last tie kept (all ties if tk == 0)
  int buf = 0;
  const bool use_k = a.top_k > 0 && (unsigned long long)a.top_k < total_fin;
  if (use_k) {
    uint32_t prefix = 0, mask = 0;
    unsigned long long need = (unsigned long long)a.top_k;
    for (int shift = 24; shift >= 0; shift -= 8, buf ^= 1) {
      if (tid < 256) sm.hist[buf][tid] = 0;
      __syncthreads();
      for (int i = tid; i < n; i += kThreads) {
        const uint32_t k = sm.keys[i];
        if (k && (k & mask) == prefix) atomicAdd(&sm.hist[buf][(k >> shift) & 255], 1ull);
      }
      unsigned long long above = 0;
      const int b = radix_pick(cl, sm, buf, need, &above);
      prefix |= (uint32_t)b << shift;
      mask |= 255u << shift;
      need -= above;
    }
    tk = prefix;
    // the first `need` ties (key == tk) in id order are kept
    unsigned long long c = 0;
    for (int i = r0; i < r1; ++i) c += sm.keys[i] == tk;
    unsigned long long tot_cta, before_cta, tot_all;
    const unsigned long long before = block_excl_scan(c, sm, &tot_cta);
    cluster_prefix(cl, sm, 2, tot_cta, &before_cta, &tot_all);
    unsigned long long run = before_cta + before;
    if (tid == 0) sm.slot[3] = kNone;
    __syncthreads();
    if (run < need && run + c >= need) {
      for (int i = r0; i < r1; ++i) {
        if (sm.keys[i] == tk && ++run == need) {
          sm.slot[3] = (unsigned long long)(i0 + i);
          break;
        }
      }
    }
    cl.sync();
    unsigned long long cut = kNone;
    for (int r = 0; r < nr; ++r) cut = min(cut, *cl.map_shared_rank(&sm.slot[3], r));
    cut_k = (long long)cut;
  }
  auto keep_k = [&](int i) -> bool {
    const uint32_t k = sm.keys[i];
    if (!k) return false;
    if (!use_k) return true;
    return k > tk || (k == tk && (long long)(i0 + i) <= cut_k);
  };
  auto weight = [&](int i) -> unsigned long long {
    const float w = expf((key_value(sm.keys[i]) - m) * a.inv_t);
    return __float2ull_rn(w * 4294967296.0f);
  };

  // 3. top-p over the survivors: threshold key tp; ties at tp kept in id
  // order until the kept mass reaches p * Z
  const bool use_p = a.top_p < 1.0f;
  uint32_t tp = 0;
  long long cut_p = -1;
  if (use_p) {
    unsigned long long zl = 0;
    for (int i = tid; i < n; i += kThreads)
      if (keep_k(i)) zl += weight(i);
    const unsigned long long z_cta = block_sum(zl, sm);
    unsigned long long bz, z;
    cluster_prefix(cl, sm, 4, z_cta, &bz, &z);
    const unsigned long long need0 = (unsigned long long)ceil((double)a.top_p * (double)z);
    unsigned long long need = need0 == 0 ? 1 : need0;
    uint32_t prefix = 0, mask = 0;
    unsigned long long above_all = 0;
    for (int shift = 24; shift >= 0; shift -= 8, buf ^= 1) {
      if (tid < 256) sm.hist[buf][tid] = 0;
      __syncthreads();
      for (int i = tid; i < n; i += kThreads) {
        const uint32_t k = sm.keys[i];
        if ((k & mask) == prefix && keep_k(i))
          atomicAdd(&sm.hist[buf][(k >> shift) & 255], weight(i));
      }
      unsigned long long above = above_all;
      const int b = radix_pick(cl, sm, buf, need, &above);
      above_all = above;
      prefix |= (uint32_t)b << shift;
      mask |= 255u << shift;
    }
    tp = prefix;
    // mass above tp is above_all; ties at tp in id order until need is reached
    unsigned long long c = 0;
    for (int i = r0; i < r1; ++i)
      if (sm.keys[i] == tp && keep_k(i)) c += weight(i);
    unsigned long long tot_cta, before_cta, tot_all;
    const unsigned long long before = block_excl_scan(c, sm, &tot_cta);
    cluster_prefix(cl, sm, 5, tot_cta, &before_cta, &tot_all);
    unsigned long long run = above_all + before_cta + before;
    if (tid == 0) sm.slot[6] = kNone;
    __syncthreads();
    if (run < need && run + c >= need) {
      for (int i = r0; i < r1; ++i) {
        if (sm.keys[i] == tp && keep_k(i)) {
          run += weight(i);
          if (run >= need) {
            sm.slot[6] = (unsigned long long)(i0 + i);
            break;
          }
        }
      }
    }
    cl.sync();
    unsigned long long cut = kNone;
    for (int r = 0; r < nr; ++r) cut = min(cut, *cl.map_shared_rank(&sm.slot[6], r));
    cut_p = (long long)cut;  // kNone (all ties) if rounding never reached the need
  }
  auto keep = [&](int i) -> bool {
    if (!keep_k(i)) return false;
    if (!use_p) return true;
    const uint32_t k = sm.keys[i];
    return k > tp || (k == tp && (long long)(i0 + i) <= cut_p);
  };

  // 4. draw: target = floor(u * Z) over the kept mass in id order
  unsigned long long c = 0;
  for (int i = r0; i < r1; ++i)
    if (keep(i)) c += weight(i);
  unsigned long long tot_cta, before_cta, z;
  const unsigned long long before = block_excl_scan(c, sm, &tot_cta);
  cluster_prefix(cl, sm, 7, tot_cta, &before_cta, &z);
  const uint32_t x = philox_first((uint32_t)a.step, (uint32_t)row, (uint32_t)(a.step >> 32), 0u,
                                  (uint32_t)a.seed, (uint32_t)(a.seed >> 32));
  const unsigned long long u24 = x >> 8;
  const unsigned long long target = (__umul64hi(u24, z) << 40) | ((u24 * z) >> 24);
  unsigned long long run = before_cta + before;
  if (tid == 0) sm.slot[8] = kNone;
  __syncthreads();
  if (run <= target && run + c > target) {
    for (int i = r0; i < r1; ++i) {
      if (keep(i)) {
        run += weight(i);
        if (run > target) {
          sm.slot[8] = (unsigned long long)(i0 + i);
          break;
        }
      }
    }
  }
  // the last kept id, for a target at the very end
  unsigned long long last = 0;
  for (int i = r1 - 1; i >= r0; --i)
    if (keep(i)) {
      last = (unsigned long long)(i0 + i) + 1;
      break;
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long t = __shfl_xor_sync(0xffffffffu, last, o);
    last = t > last ? t : last;
  }
  if (lane == 0) sm.warp_part[warp] = last;
  __syncthreads();
  if (tid == 0) {
    unsigned long long l = 0;
    for (int w = 0; w < kWarps; ++w) l = max(l, sm.warp_part[w]);
    sm.slot[9] = l;
  }
  cl.sync();
  if (rank == 0 && tid == 0) {
    unsigned long long pick = kNone, lastk = 0;
    for (int r = 0; r < nr; ++r) {
      pick = min(pick, *cl.map_shared_rank(&sm.slot[8], r));
      lastk = max(lastk, *cl.map_shared_rank(&sm.slot[9], r));
    }
    if (pick == kNone) pick = lastk ? lastk - 1 : 0;
    a.out[row] = (int32_t)pick;
  }
  cl.sync();  // no CTA leaves while another may still read its shared memory
}

}  // namespace samp

size_t sample_smem_bytes(int V, int nr) {
  const int chunk = (V + nr - 1) / nr;
  return sizeof(samp::Smem) + (size_t)chunk * sizeof(uint32_t);
}

// Cluster size per row: the smallest of 2, 4, 8 whose key slices fit.
int sample_cluster(int V) {
  for (int nr : {2, 4, 8})
    if (sample_smem_bytes(V, nr) <= 200 * 1024) return nr;
  return 0;
}

cudaError_t launch_sample(const float* logits, int rows, int V, float temperature, int top_k,
                          float top_p, unsigned long long seed, unsigned long long step,
                          int32_t* out, cudaStream_t st) {
  const int nr = sample_cluster(V);
  if (!nr) return cudaErrorInvalidValue;
  samp::Args a;
  a.logits = logits;
  a.V = V;
  a.chunk = (V + nr - 1) / nr;
  a.inv_t = 1.0f / temperature;
  a.top_k = top_k;
  a.top_p = top_p;
  a.seed = seed;
  a.step = step;
  a.out = out;
  const size_t smem = sample_smem_bytes(V, nr);
  cudaError_t e = cudaFuncSetAttribute(samp::sample_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(samp::sample_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rows * nr);
  cfg.blockDim = dim3(samp::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = nr;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launches();
  e = cudaLaunchKernelEx(&cfg, samp::sample_kernel, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fs
