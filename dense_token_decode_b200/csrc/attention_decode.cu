// Split-KV causal GQA attention for decode batches and short prefill chunks
// over the paged bf16 cache (flash-decoding): every row attends its own
// context 0..pos, and the context is cut into splits of whole 64-position
// pages so that a batch of long sequences fills the GPU.
//
// One CTA of 4 warps per (split, kv head, row). The G = nq / nkv query heads
// of the group share every K/V load. A warp owns whole pages of the split
// and walks them 8 keys at a time: each lane holds d/32 dimensions of the 8
// K and V rows (coalesced 256-byte rows), the 8 x G partial dot products are
// reduced across the warp by a transposing butterfly (one value per lane pair
// at the end), and the online softmax runs in the exp2 domain with warp-
// uniform per-head max / sum. The 4 warps merge in shared memory and the CTA
// writes one (max, sum, o[d]) partial per query head; a second kernel merges
// the splits (log-sum-exp weights) into o.
//
// The work is HBM-bound: K and V bytes of every attended position are read
// once per kv head, 2 x 2 x d bytes per (row, kv head, position).
#include <algorithm>

#include "fs_internal.h"

namespace fs {

constexpr int kDecAttnRows = 128;   // rows one call may cover
constexpr int kDecAttnSplits = 32;  // splits per (row, kv head) at most

namespace {

constexpr int kWarps = 4;
constexpr int kGroupKeys = 8;

struct DecParams {
  const float* q;  // [rows][nq][D]
  float* part;     // [rows][nq][splits][D + 2]: o (unnormalised), max, sum
  float* o;        // [rows][nq * D]
  RowMap map;
  KVView kv;
  int layer, nq, nkv, splits, pages_per_split;
  float scale_log2;
};

__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// E consecutive bf16 values (E = 2 or 4) as fp32.
template <int E>
__device__ __forceinline__ void load_row(const __nv_bfloat16* p, float (&x)[E]) {
  if constexpr (E == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    x[0] = bf_lo(u.x); x[1] = bf_hi(u.x); x[2] = bf_lo(u.y); x[3] = bf_hi(u.y);
  } else {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
    x[0] = bf_lo(u); x[1] = bf_hi(u);
  }
}

// Transposing butterfly: NV partial sums per lane -> the full sum of value
// v = lane >> (5 - log2 NV) in every lane (NV a power of two, 2..32).
template <int NV>
__device__ __forceinline__ float reduce_transpose(float (&v)[NV], int lane) {
  int w = NV / 2, mask = 16;
#pragma unroll
  for (; w >= 1; w >>= 1, mask >>= 1) {
    const bool upper = (lane & mask) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float send = upper ? v[i] : v[i + w];
      const float keep = upper ? v[i + w] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
    }
  }
  float s = v[0];
#pragma unroll
  for (; mask >= 1; mask >>= 1) s += __shfl_xor_sync(0xffffffffu, s, mask);
  return s;
}

template <int D, int G>
__global__ void __launch_bounds__(kWarps * 32) attention_decode_kernel(const DecParams p) {
  pdl_trigger();
  pdl_wait();
  constexpr int E = D / 32;              // dims per lane
  constexpr int NV = kGroupKeys * G;     // partial scores per lane per group
  constexpr int LOG_NV = NV == 8 ? 3 : NV == 16 ? 4 : 5;
  constexpr int SH = 5 - LOG_NV;         // lane >> SH = value index
  static_assert(NV == 8 || NV == 16 || NV == 32, "group size");
  __shared__ float s_m[kWarps][G], s_l[kWarps][G];
  __shared__ float s_o[kWarps][G][D];

  const int split = blockIdx.x, g = blockIdx.y, r = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const RowInfo ri = p.map.get(r);
  const int n_pages = ri.pos / kPage + 1;
  const int pg0 = split * p.pages_per_split;
  const int pg1 = min(pg0 + p.pages_per_split, n_pages);

  float q[G][E];
#pragma unroll
  for (int j = 0; j < G; ++j)
#pragma unroll
    for (int e = 0; e < E; ++e)
      q[j][e] = p.q[((size_t)r * p.nq + g * G + j) * D + lane * E + e] * p.scale_log2;

  float m[G], l[G], acc[G][E];
#pragma unroll
  for (int j = 0; j < G; ++j) {
    m[j] = -INFINITY;
    l[j] = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[j][e] = 0.f;
  }

  // my (key, head) slot after the reduction
  const int my_v = lane >> SH;
  const int my_k = my_v / G, my_j = my_v % G;

  for (int pg = pg0 + warp; pg < pg1; pg += kWarps) {
    const size_t base = p.kv.offset(p.layer, ri.seq, pg * kPage, g);
    for (int kb = 0; kb < kPage; kb += kGroupKeys) {
      const int key0 = pg * kPage + kb;
      if (key0 > ri.pos) break;
      float kr[kGroupKeys][E], vr[kGroupKeys][E];
#pragma unroll
      for (int k = 0; k < kGroupKeys; ++k) {
        load_row<E>(p.kv.k + base + (size_t)(kb + k) * D + lane * E, kr[k]);
        load_row<E>(p.kv.v + base + (size_t)(kb + k) * D + lane * E, vr[k]);
      }
      float part[NV];
#pragma unroll
      for (int k = 0; k < kGroupKeys; ++k)
#pragma unroll
        for (int j = 0; j < G; ++j) {
          float s = 0.f;
#pragma unroll
          for (int e = 0; e < E; ++e) s = fmaf(q[j][e], kr[k][e], s);
          part[k * G + j] = s;
        }
      float sc = reduce_transpose<NV>(part, lane);
      if (key0 + my_k > ri.pos) sc = -INFINITY;
      // per-head max over the 8 keys: lanes with the same head differ in the key bits
      float gm = sc;
#pragma unroll
      for (int b = SH + (G == 1 ? 0 : G == 2 ? 1 : 2); b < 5; ++b)
        gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, 1 << b));
      float m_new[G], alpha[G];
#pragma unroll
      for (int j = 0; j < G; ++j) {
        const float gmj = __shfl_sync(0xffffffffu, gm, j << SH);
        m_new[j] = fmaxf(m[j], gmj);  // key0 <= pos: at least one finite score
        alpha[j] = exp2f(m[j] - m_new[j]);
      }
      float mj = m_new[0];
#pragma unroll
      for (int j = 1; j < G; ++j)
        if (my_j == j) mj = m_new[j];
      const float pv = exp2f(sc - mj);
      float gs = pv;
#pragma unroll
      for (int b = SH + (G == 1 ? 0 : G == 2 ? 1 : 2); b < 5; ++b)
        gs += __shfl_xor_sync(0xffffffffu, gs, 1 << b);
#pragma unroll
      for (int j = 0; j < G; ++j) {
        l[j] = l[j] * alpha[j] + __shfl_sync(0xffffffffu, gs, j << SH);
        m[j] = m_new[j];
#pragma unroll
        for (int e = 0; e < E; ++e) acc[j][e] *= alpha[j];
      }
#pragma unroll
      for (int k = 0; k < kGroupKeys; ++k)
#pragma unroll
        for (int j = 0; j < G; ++j) {
          const float pk = __shfl_sync(0xffffffffu, pv, (k * G + j) << SH);
#pragma unroll
          for (int e = 0; e < E; ++e) acc[j][e] = fmaf(pk, vr[k][e], acc[j][e]);
        }
    }
  }

  // merge the warps of the CTA
#pragma unroll
  for (int j = 0; j < G; ++j) {
    if (lane == 0) {
      s_m[warp][j] = m[j];
      s_l[warp][j] = l[j];
    }
#pragma unroll
    for (int e = 0; e < E; ++e) s_o[warp][j][lane * E + e] = acc[j][e];
  }
  __syncthreads();
  for (int t = threadIdx.x; t < G * D; t += kWarps * 32) {
    const int j = t / D, c = t % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, s_m[w][j]);
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float f = s_m[w][j] == -INFINITY ? 0.f : exp2f(s_m[w][j] - M);
        L += s_l[w][j] * f;
        O += s_o[w][j][c] * f;
      }
    }
    float* dst = p.part + (((size_t)r * p.nq + g * G + j) * p.splits + split) * (D + 2);
    dst[c] = O;
    if (c == 0) {
      dst[D] = M;
      dst[D + 1] = L;
    }
  }
}

// o[r, h, :] = sum_s w_s o_s / sum_s w_s l_s, w_s = 2^(m_s - max m).
template <int D>
__global__ void __launch_bounds__(D) attention_merge_kernel(const DecParams p) {
  pdl_trigger();
  pdl_wait();
  const int h = blockIdx.x, r = blockIdx.y, c = threadIdx.x;
  const float* src = p.part + ((size_t)r * p.nq + h) * p.splits * (D + 2);
  float M = -INFINITY;
  for (int s = 0; s < p.splits; ++s) M = fmaxf(M, src[(size_t)s * (D + 2) + D]);
  float L = 0.f, O = 0.f;
  for (int s = 0; s < p.splits; ++s) {
    const float ms = src[(size_t)s * (D + 2) + D];
    if (ms == -INFINITY) continue;
    const float f = exp2f(ms - M);
    L += src[(size_t)s * (D + 2) + D + 1] * f;
    O += src[(size_t)s * (D + 2) + c] * f;
  }
  p.o[((size_t)r * p.nq + h) * D + c] = O / L;
}

template <int D, int G>
cudaError_t launch_dec(const DecParams& p, int rows, cudaStream_t st) {
  dim3 grid(p.splits, p.nkv, rows);
  count_launches(2);
  cudaError_t e = launch_pdl(attention_decode_kernel<D, G>, grid, dim3(kWarps * 32), 0, st, p);
  if (e != cudaSuccess) return e;
  return launch_pdl(attention_merge_kernel<D>, dim3(p.nq, rows), dim3(D), 0, st, p);
}

}  // namespace

bool attention_decode_supported(const Shape& s, int rows) {
  const int G = s.nkv > 0 ? s.nq / s.nkv : 0;
  return rows >= 1 && rows <= kDecAttnRows && (s.d == 64 || s.d == 128) &&
         s.nq % s.nkv == 0 && (G == 1 || G == 2 || G == 4);
}

size_t attention_decode_part_floats(const Shape& s) {
  return (size_t)kDecAttnRows * s.nq * kDecAttnSplits * (s.d + 2);
}

// Split count: enough CTAs to cover the SMs a few times over, whole pages per
// split, at most kDecAttnSplits. `max_pos` is the largest position of the rows.
cudaError_t launch_attention_decode(const float* q, int rows, const RowMap& map, int max_pos,
                                    const Shape& s, KVView kv, int layer, float* part, float* o,
                                    int num_sms, cudaStream_t st) {
  if (!attention_decode_supported(s, rows)) return cudaErrorInvalidValue;
  const int pages = max_pos / kPage + 1;
  const int want = (8 * num_sms + rows * s.nkv - 1) / (rows * s.nkv);  // splits wanted
  int splits = std::min(std::min(pages, kDecAttnSplits), std::max(1, want));
  const int pps = (pages + splits - 1) / splits;
  splits = (pages + pps - 1) / pps;
  DecParams p;
  p.q = q;
  p.part = part;
  p.o = o;
  p.map = map;
  p.kv = kv;
  p.layer = layer;
  p.nq = s.nq;
  p.nkv = s.nkv;
  p.splits = splits;
  p.pages_per_split = pps;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)s.d);
  const int G = s.nq / s.nkv;
  if (s.d == 128) {
    if (G == 1) return launch_dec<128, 1>(p, rows, st);
    if (G == 2) return launch_dec<128, 2>(p, rows, st);
    return launch_dec<128, 4>(p, rows, st);
  }
  if (G == 1) return launch_dec<64, 1>(p, rows, st);
  if (G == 2) return launch_dec<64, 2>(p, rows, st);
  return launch_dec<64, 4>(p, rows, st);
}

}  // namespace fs
