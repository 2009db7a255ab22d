// Lightning Indexer scores and per-query top-k selection.
//
// Method: "DeepSeek-V4" doc, "Hybrid attention (§2.3)" CSA item — the Lightning Indexer
// (eqs. 13-17) scores each query against the compressed pool and keeps the top
// index_topk entries (eq. 17); "Attention mask layout" — -1 sentinels while fewer
// entries are ready.  "DeepSeek-V3.2" doc, "DeepSeek Sparse Attention (DSA)" — a
// low-head-count scorer with per-head weights; since the Hadamard rotation of the
// reference indexer is orthogonal, the scores are computed directly.
//
// Score kernel (CUDA cores, fp32 accumulation): a CTA owns 128 pool entries (one per
// thread) and 64 (query, head) rows.  The entry tile is staged once in shared memory,
// each thread keeps its 64 dot products in registers, and the ReLU / head weights /
// head sum happen in the epilogue, so the per-query score row is the only output.
//
// Top-k kernel: one CTA per query row.  Radix select over an order-preserving 32-bit
// key of the fp32 score (4 passes of 8 bits) finds the K-th largest score T; every
// entry above T is kept, and of the entries equal to T the lowest indices are kept
// (the tie rule).  The kept entries are written in ascending entry order, which also
// gives the attention gathers increasing addresses.
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace dsv4 {

namespace {

constexpr int kTileW = 128;  // entries per score CTA
constexpr int kRowsQH = 64;  // (query, head) rows per score CTA

template <typename T, int NI, int CI>
__global__ void __launch_bounds__(kTileW) indexer_scores_kernel(IndexerArgs a, int64_t row0, int64_t row1) {
  constexpr int QB = kRowsQH / NI;  // queries per CTA
  extern __shared__ float smem[];
  float* qs = smem;                               // [64][CI]
  float* ks = qs + kRowsQH * CI;                  // [128][CI+1]
  __shared__ float ws[kRowsQH];
  __shared__ int vis_s[QB];
  __shared__ int maxvis_s;

  const int tile = blockIdx.x;
  const int64_t rbase = row0 + (int64_t)blockIdx.y * QB;
  const int tid = threadIdx.x;

  if (tid == 0) maxvis_s = 0;
  __syncthreads();
  if (tid < QB) {
    const int64_t row = rbase + tid;
    int v = 0;
    if (row < row1) {
      const int s = (int)(row % a.Sq);
      const int t = query_cache_index(a.q_index, row, s);
      v = visible_entries(t, a.m, a.P_cap);
    }
    vis_s[tid] = v;
    atomicMax(&maxvis_s, v);
  }
  __syncthreads();
  const int w0 = tile * kTileW;
  if (w0 >= maxvis_s) return;  // nothing in this tile is visible to any query of the CTA

  // stage query rows and head weights (rows past row1 are zero)
  const T* qI = static_cast<const T*>(a.qI);
  for (int i = tid; i < kRowsQH * CI; i += kTileW) {
    const int r = i / CI;
    const int64_t row = rbase + r / NI;
    qs[i] = row < row1 ? to_f32<T>(qI[(rbase * NI) * CI + i]) : 0.f;
  }
  if (tid < kRowsQH) {
    const int64_t row = rbase + tid / NI;
    ws[tid] = row < row1 ? a.wI[rbase * NI + tid] : 0.f;
  }
  __syncthreads();

  // The rows of a CTA may belong to several sequences (always when Sq < QB): the entry
  // tile is staged and scored once per distinct sequence.  Entries past P_cap are zero.
  const int64_t seq_first = rbase / a.Sq;
  const int64_t last_row = (rbase + QB - 1 < row1 ? rbase + QB - 1 : row1 - 1);
  const int64_t seq_last = last_row / a.Sq;
  const T* poolI = static_cast<const T*>(a.poolI);
  for (int64_t sq = seq_first; sq <= seq_last; ++sq) {
    __syncthreads();
    for (int i = tid; i < kTileW * CI; i += kTileW) {
      const int e = i / CI, d = i % CI;
      const int w = w0 + e;
      ks[e * (CI + 1) + d] = w < a.P_cap ? to_f32<T>(poolI[((int64_t)sq * a.P_cap + w) * CI + d]) : 0.f;
    }
    __syncthreads();

    float acc[kRowsQH];
#pragma unroll
    for (int i = 0; i < kRowsQH; ++i) acc[i] = 0.f;
    const float* krow = ks + tid * (CI + 1);
#pragma unroll 2
    for (int d = 0; d < CI; d += 4) {
      const float k0 = krow[d], k1 = krow[d + 1], k2 = krow[d + 2], k3 = krow[d + 3];
#pragma unroll
      for (int i = 0; i < kRowsQH; ++i) {
        const float4 qv = *reinterpret_cast<const float4*>(qs + i * CI + d);
        acc[i] = fmaf(k0, qv.x, acc[i]);
        acc[i] = fmaf(k1, qv.y, acc[i]);
        acc[i] = fmaf(k2, qv.z, acc[i]);
        acc[i] = fmaf(k3, qv.w, acc[i]);
      }
    }
    const int w = w0 + tid;
#pragma unroll
    for (int q = 0; q < QB; ++q) {
      float sc = 0.f;
#pragma unroll
      for (int h = 0; h < NI; ++h) sc = fmaf(ws[q * NI + h], fmaxf(acc[q * NI + h], 0.f), sc);
      const int64_t row = rbase + q;
      if (row < row1 && row / a.Sq == sq && w < vis_s[q]) a.scores[(row - row0) * a.P_cap + w] = sc;
    }
  }
}

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0u) u = 0u;  // -0 and +0 are the same score
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kTopkBins = 4096;        // radix digits of 12 bits
constexpr int kTopkSmemKeys = 40960;   // keys cached in shared memory (160 KB)

constexpr int kTopkListBytes = 20480;  // uncached rows: the warps' lists of entries at or above the threshold digit
constexpr uint32_t kListDigit = 0x80000000u;  // list entry flag: the entry's key is in the threshold digit

// The keys of entries base + u * stride (u < 8), 0 at or past `end`: all eight loads are
// issued before any is used, so a pass over a long row costs a few memory round trips per
// eight keys of each thread instead of one per key.
__device__ __forceinline__ void row_keys8(uint32_t (&k)[8], const uint32_t* keys, const float* sc, bool cached,
                                          int base, int stride, int end) {
  if (cached) {
#pragma unroll
    for (int u = 0; u < 8; ++u) k[u] = base + u * stride < end ? keys[base + u * stride] : 0u;
  } else {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = base + u * stride < end ? sc[base + u * stride] : 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) k[u] = order_key(v[u]);
  }
}

// The keys of the eight consecutive entries e0 .. e0 + 7 (e0 a multiple of 8), 0 at or past
// `end`: two 16-byte loads when `vec` (every row starts on 16 bytes and holds a multiple of 4
// entries, so a vector that starts below `end` stays inside the row), else eight 4-byte ones.
__device__ __forceinline__ void row_run8(uint32_t (&k)[8], const float* sc, bool vec, int e0, int end) {
  float v[8];
  if (vec) {
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 x = e0 < end ? *reinterpret_cast<const float4*>(sc + e0) : z;
    const float4 y = e0 + 4 < end ? *reinterpret_cast<const float4*>(sc + e0 + 4) : z;
    v[0] = x.x;
    v[1] = x.y;
    v[2] = x.z;
    v[3] = x.w;
    v[4] = y.x;
    v[5] = y.y;
    v[6] = y.z;
    v[7] = y.w;
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = e0 + j < end ? sc[e0 + j] : 0.f;
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) k[j] = order_key(v[j]);
}

// Finds the digit holding the need-th largest key of a histogram (digits scanned from the
// top): *bin = that digit, *rest = how many keys of it are still needed, *cnt = its count.
// Thread t owns the descending run of digits [top - BPT + 1, top], top = kTopkBins-1-t*BPT.
template <int NT>
__device__ __forceinline__ void find_digit(const uint32_t* hist, int need, int* wsum, int* bin, int* rest,
                                           int* cnt_out) {
  constexpr int BPT = kTopkBins / NT;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int top = kTopkBins - 1 - tid * BPT;
  int cnt[BPT];
  int sum = 0;
#pragma unroll
  for (int k = 0; k < BPT; ++k) {
    cnt[k] = (int)hist[top - k];
    sum += cnt[k];
  }
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = lane < NT / 32 ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += n;
    }
    if (lane < NT / 32) wsum[lane] = v;
  }
  __syncthreads();
  incl += warp > 0 ? wsum[warp - 1] : 0;
  const int excl = incl - sum;
  if (excl < need && need <= incl) {
    int run = excl;
#pragma unroll
    for (int k = 0; k < BPT; ++k) {
      if (run < need && need <= run + cnt[k]) {
        *bin = top - k;
        *rest = need - run;
        *cnt_out = cnt[k];
      }
      run += cnt[k];
    }
  }
  __syncthreads();
}

// One warp lists, in entry order, the entries e of [lo, hi) whose key's top digit is at least
// b1: list[p] = e, with kListDigit set when the digit is b1 (entries past kCap are counted,
// not stored).  Lane l takes the run of eight entries base + 8l .. base + 8l + 7 and a scan of
// the lanes' counts places each run's entries.  With `track`, each lane also counts its keys
// of digit b1 and keeps their least and greatest.  Returns the segment's number of listed
// entries (the same in every lane).
template <int kCap>
__device__ __forceinline__ int list_segment(const float* sc, bool vec, int lo, int hi, uint32_t b1, bool track,
                                            uint32_t* list, int& n_eq, uint32_t& kmin, uint32_t& kmax) {
  const int lane = threadIdx.x & 31;
  int len = 0;
  for (int base = lo; base < hi; base += 32 * 8) {
    const int e0 = base + lane * 8;
    uint32_t kk[8];
    row_run8(kk, sc, vec, e0, hi);
    uint32_t selm = 0u, digm = 0u;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t dg = kk[j] >> 20;
      const bool sel = e0 + j < hi && dg >= b1;
      selm |= (uint32_t)sel << j;
      digm |= (uint32_t)(dg == b1) << j;
      if (track && sel && dg == b1) {
        n_eq += 1;
        kmin = min(kmin, kk[j]);
        kmax = max(kmax, kk[j]);
      }
    }
    const int c = __popc(selm);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    if (len < kCap) {
      int pos = len + incl - c;
      for (uint32_t m = selm; m != 0u; m &= m - 1u, ++pos) {
        const int j = __ffs(m) - 1;
        if (pos < kCap) list[pos] = (uint32_t)(e0 + j) | ((digm >> j) & 1u ? kListDigit : 0u);
      }
    }
    len += __shfl_sync(0xffffffffu, incl, 31);
  }
  return len;
}

// Per-query top-k by radix select over order-preserving keys: a 12-bit digit histogram
// while the row is loaded, then 12 and 8 more bits over the keys that still match the
// selected prefix (skipped once the threshold digit holds exactly the keys still needed).
// Output: the kept entries in ascending entry order, then -1.
// A row not cached in shared memory (cache_keys == 0) reads its scores twice: the histogram,
// then one pass in which each warp lists, in entry order, the entries of its segment of the
// row whose key is at or above the threshold digit (a flag marks those in that digit).  The
// remaining digits, the counts and the ordered write then go over the lists alone (the keys
// of the listed threshold-digit entries are read again).  A list that would outgrow its share
// of shared memory sends the row to the passes over the whole row; when the threshold digit
// holds one value only (a long run of equal scores, such as the exact zeros that ReLU leaves
// in a one-head indexer), that value is the whole prefix and the counts come from the same
// pass.  A row of at least 4 topk entries first takes its threshold digit from an eighth of
// its entries instead of the full histogram (see below), so it reads its scores about 1.1
// times when that works.
template <int NT>
__global__ void __launch_bounds__(NT, NT <= 256 ? 6 : 1) topk_kernel(IndexerArgs a, int64_t row0, int cache_keys) {
  extern __shared__ __align__(16) uint32_t keys[];  // the row's keys (cached rows) or the warps' lists
  __shared__ uint32_t hist[kTopkBins];
  __shared__ int wsum[NT / 32];
  __shared__ int s_bin, s_rest, s_cnt, s_over, s_len, s_eq;
  __shared__ uint32_t s_kmin, s_kmax;
  __shared__ int wcnt_gt[NT / 32], wcnt_eq[NT / 32];
  constexpr int kWarps = NT / 32;
  constexpr int kCap = kTopkListBytes / 4 / kWarps;  // entries of one warp's list

  const int64_t row = row0 + blockIdx.x;
  const int s = (int)(row % a.Sq);
  const int t = query_cache_index(a.q_index, row, s);
  const int vis = visible_entries(t, a.m, a.P_cap);
  const int K = a.topk;
  int32_t* out = a.idx + row * (int64_t)K;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned below = (1u << lane) - 1u;

  if (vis <= K) {
    for (int i = tid; i < K; i += NT) out[i] = i < vis ? i : -1;
    return;
  }
  const float* sc = a.scores + (int64_t)blockIdx.x * a.P_cap;
  const bool cached = vis <= cache_keys;  // keys kept in shared memory
  const bool uncached = !cached && cache_keys == 0;
  const bool vec = (a.P_cap & 3) == 0 && (reinterpret_cast<uintptr_t>(a.scores) & 15) == 0;
  const int seg = ((vis + kWarps - 1) / kWarps + 7) & ~7;  // warp segments start on 8 entries
  const int lo = min(vis, warp * seg), hi = min(vis, lo + seg);
  uint32_t* list = keys + warp * kCap;
  uint32_t prefix = 0u, mask = 0xFFF00000u;
  int need = 0;
  int n_gt = 0, n_eq = 0;  // this warp segment's keys above / equal to the final prefix
  int len = 0;             // entries of this warp's segment in its list
  bool counted = false, listed = false;
  bool allcand = false;  // the lists hold candidates of a sampled threshold: every key is compared

  // A long uncached row first takes its threshold digit from a sample (the first 32 entries of
  // every 256), placed so that about 5/4 topk entries of the row lie at or above it, and lists
  // them.  The selection is then exact over the lists when they hold at least topk entries and
  // fit; when they overflow only because the threshold digit is one long run of a value that
  // holds the topk-th key, the counts are done as below; otherwise the row starts again on the
  // general path.
  if (uncached && vis >= 4 * K) {
    for (int i = tid; i < kTopkBins; i += NT) hist[i] = 0u;
    if (tid == 0) {
      s_over = 0;
      s_len = 0;
      s_eq = 0;
      s_kmin = 0xFFFFFFFFu;
      s_kmax = 0u;
    }
    __syncthreads();
    for (int c0 = warp; c0 * 256 < vis; c0 += kWarps * 8) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int e = (c0 + u * kWarps) * 256 + lane;
        v[u] = e < vis ? sc[e] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if ((c0 + u * kWarps) * 256 + lane < vis) atomicAdd(&hist[order_key(v[u]) >> 20], 1u);
    }
    __syncthreads();
    const int ns = (vis >> 8) * 32 + min(32, vis & 255);  // sampled entries
    const int ks = min(ns, (int)((int64_t)K * ns * 5 / (4 * (int64_t)vis)) + 32);
    find_digit<NT>(hist, ks, wsum, &s_bin, &s_rest, &s_cnt);
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
    int eqc = 0;
    len = list_segment<kCap>(sc, vec, lo, hi, (uint32_t)s_bin, true, list, eqc, kmin, kmax);
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    eqc = __reduce_add_sync(0xffffffffu, eqc);
    if (lane == 0) {
      if (len > kCap) s_over = 1;
      atomicAdd(&s_len, len);
      atomicAdd(&s_eq, eqc);
      if (kmin <= kmax) {
        atomicMin(&s_kmin, kmin);
        atomicMax(&s_kmax, kmax);
      }
    }
    __syncthreads();
    const int tot = s_len, tot_gt = s_len - s_eq;
    if (s_over == 0 && tot >= K) {
      listed = true;
      allcand = true;
    } else if (s_over != 0 && tot_gt < K && tot >= K && s_kmin == s_kmax) {
      prefix = s_kmin;
      mask = 0xFFFFFFFFu;
      need = K - tot_gt;
      n_gt = len - eqc;
      n_eq = eqc;
      counted = true;
    }
    __syncthreads();  // every thread has read the shared words before the general path resets them
  }
  if (!listed && !counted) {
    for (int i = tid; i < kTopkBins; i += NT) hist[i] = 0u;
    __syncthreads();
    // each thread takes runs of eight consecutive entries
    for (int e0 = tid * 8; e0 < vis; e0 += NT * 8) {
      uint32_t kk[8];
      row_run8(kk, sc, vec, e0, vis);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (e0 + j < vis) {
          if (cached) keys[e0 + j] = kk[j];
          atomicAdd(&hist[kk[j] >> 20], 1u);
        }
      }
    }
    __syncthreads();
    find_digit<NT>(hist, K, wsum, &s_bin, &s_rest, &s_cnt);
    prefix = (uint32_t)s_bin << 20;
    need = s_rest;
    len = 0;
    if (uncached) {
      // a list can outgrow its share only when the entries to list outnumber one share
      const bool track = K - need + s_cnt > kCap;
      if (tid == 0) {
        s_over = 0;
        s_kmin = 0xFFFFFFFFu;
        s_kmax = 0u;
      }
      __syncthreads();
      uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
      len = list_segment<kCap>(sc, vec, lo, hi, (uint32_t)s_bin, track, list, n_eq, kmin, kmax);
      if (lane == 0 && len > kCap) s_over = 1;
      if (track) {
        kmin = __reduce_min_sync(0xffffffffu, kmin);
        kmax = __reduce_max_sync(0xffffffffu, kmax);
        n_eq = __reduce_add_sync(0xffffffffu, n_eq);
        if (lane == 0 && kmin <= kmax) {
          atomicMin(&s_kmin, kmin);
          atomicMax(&s_kmax, kmax);
        }
      }
      __syncthreads();
      listed = s_over == 0;
      if (!listed && s_cnt != need && s_kmin == s_kmax) {
        // the threshold digit holds one value: it is the whole prefix, and the counts are done
        prefix = s_kmin;
        mask = 0xFFFFFFFFu;
        n_gt = len - n_eq;
        counted = true;
      } else {
        n_eq = 0;
      }
    }
  }
  if (listed) {
    if (allcand) {
      // the top digit over every listed entry
      for (int i = tid; i < kTopkBins; i += NT) hist[i] = 0u;
      __syncthreads();
      for (int p = lane; p < len; p += 32) atomicAdd(&hist[order_key(sc[list[p] & ~kListDigit]) >> 20], 1u);
      __syncthreads();
      find_digit<NT>(hist, K, wsum, &s_bin, &s_rest, &s_cnt);
      prefix = (uint32_t)s_bin << 20;
      need = s_rest;
    }
    // the remaining 12 and 8 bits over the listed entries of the threshold digit (every
    // listed entry after a sampled threshold)
    for (int pass = 1; pass < 3 && s_cnt != need; ++pass) {
      const int shift = pass == 1 ? 8 : 0;
      const uint32_t dmask = pass == 1 ? 0xFFFu : 0xFFu;
      for (int i = tid; i < kTopkBins; i += NT) hist[i] = 0u;
      __syncthreads();
      for (int p = lane; p < len; p += 32) {
        const uint32_t e = list[p];
        if (allcand || (e & kListDigit)) {
          const uint32_t k = order_key(sc[e & ~kListDigit]);
          if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & dmask], 1u);
        }
      }
      __syncthreads();
      find_digit<NT>(hist, need, wsum, &s_bin, &s_rest, &s_cnt);
      prefix |= (uint32_t)s_bin << shift;
      mask |= dmask << shift;
      need = s_rest;
    }
    // this segment's listed keys above / equal to the final prefix (entries outside the
    // threshold digit are above it)
    for (int p = lane; p < len; p += 32) {
      const uint32_t e = list[p];
      if (allcand || (e & kListDigit)) {
        const uint32_t k = order_key(sc[e & ~kListDigit]) & mask;
        n_gt += k > prefix;
        n_eq += k == prefix;
      } else {
        n_gt += 1;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      n_gt += __shfl_xor_sync(0xffffffffu, n_gt, o);
      n_eq += __shfl_xor_sync(0xffffffffu, n_eq, o);
    }
    counted = true;
  }
  for (int pass = 1; pass < 3 && s_cnt != need && !counted; ++pass) {
    const int shift = pass == 1 ? 8 : 0;
    const uint32_t dmask = pass == 1 ? 0xFFFu : 0xFFu;
    for (int i = tid; i < kTopkBins; i += NT) hist[i] = 0u;
    __syncthreads();
    for (int base = tid; base < vis; base += NT * 8) {
      uint32_t kk[8];
      row_keys8(kk, keys, sc, cached, base, NT, vis);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (base + u * NT < vis && (kk[u] & mask) == prefix) atomicAdd(&hist[(kk[u] >> shift) & dmask], 1u);
    }
    __syncthreads();
    find_digit<NT>(hist, need, wsum, &s_bin, &s_rest, &s_cnt);
    prefix |= (uint32_t)s_bin << shift;
    mask |= dmask << shift;
    need = s_rest;
  }
  // Keep every key whose masked value is above `prefix` and the `need` lowest-index keys
  // equal to it (all of them when the loop stopped early), in ascending entry order: each
  // warp owns a contiguous segment of the row; per-warp counts, a scan over warps, then
  // ordered writes.
  if (!counted) {
    for (int base = lo + lane; base < hi; base += 32 * 8) {
      uint32_t kk[8];
      row_keys8(kk, keys, sc, cached, base, 32, hi);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t k = kk[u] & mask;
        const bool in = base + u * 32 < hi;
        n_gt += in && k > prefix;
        n_eq += in && k == prefix;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      n_gt += __shfl_xor_sync(0xffffffffu, n_gt, o);
      n_eq += __shfl_xor_sync(0xffffffffu, n_eq, o);
    }
  }
  if (lane == 0) {
    wcnt_gt[warp] = n_gt;
    wcnt_eq[warp] = n_eq;
  }
  __syncthreads();
  int gt_before = 0, eq_before = 0;
  for (int w = 0; w < warp; ++w) {
    gt_before += wcnt_gt[w];
    eq_before += wcnt_eq[w];
  }
  // output slot of an entry = (kept entries before it): kept-greater before it plus the kept
  // ties before it (ties are kept while their rank among ties is below `need`)
  int pos_gt = gt_before, pos_eq = eq_before;
  const int gt_end = gt_before + wcnt_gt[warp];
  if (listed) {
    for (int base = 0; base < len; base += 32) {
      const int p = base + lane;
      const uint32_t e = p < len ? list[p] : 0u;
      const bool dig = allcand || (e & kListDigit) != 0u;
      const uint32_t k = dig ? order_key(sc[e & ~kListDigit]) & mask : 0u;
      const bool gt = p < len && (!dig || k > prefix);
      const bool eq = p < len && dig && k == prefix;
      const unsigned bgt = __ballot_sync(0xffffffffu, gt), beq = __ballot_sync(0xffffffffu, eq);
      const int my_eq_rank = pos_eq + __popc(beq & below);
      const int slot = pos_gt + __popc(bgt & below) + min(my_eq_rank, need);
      if ((gt || (eq && my_eq_rank < need)) && slot < K) out[slot] = (int)(e & ~kListDigit);
      pos_gt += __popc(bgt);
      pos_eq += __popc(beq);
    }
    return;
  }
  // A warp stops once its segment's greater keys are all written and the kept ties are all
  // behind it (a long run of one value keeps only its first `need` entries).
  for (int base = lo; base < hi && (pos_gt < gt_end || pos_eq < need); base += 32 * 8) {
    uint32_t kk[8];
    row_keys8(kk, keys, sc, cached, base + lane, 32, hi);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = base + u * 32 + lane;
      const uint32_t k = kk[u] & mask;
      const bool gt = i < hi && k > prefix;
      const bool eq = i < hi && k == prefix;
      const unsigned bgt = __ballot_sync(0xffffffffu, gt), beq = __ballot_sync(0xffffffffu, eq);
      const int my_eq_rank = pos_eq + __popc(beq & below);
      const int slot = pos_gt + __popc(bgt & below) + min(my_eq_rank, need);
      if ((gt || (eq && my_eq_rank < need)) && slot < K) out[slot] = i;
      pos_gt += __popc(bgt);
      pos_eq += __popc(beq);
    }
  }
}

template <typename T, int NI, int CI>
cudaError_t launch_scores_t(const IndexerArgs& a, int64_t r0, int64_t r1, cudaStream_t st) {
  constexpr int QB = kRowsQH / NI;
  const size_t smem = (size_t)(kRowsQH * CI + kTileW * (CI + 1)) * sizeof(float);
  cudaFuncSetAttribute(indexer_scores_kernel<T, NI, CI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)smem);
  dim3 grid((a.P_cap + kTileW - 1) / kTileW, (unsigned)((r1 - r0 + QB - 1) / QB));
  indexer_scores_kernel<T, NI, CI><<<grid, kTileW, smem, st>>>(a, r0, r1);
  note_launch();
  return cudaGetLastError();
}

template <typename T, int CI>
cudaError_t launch_scores_ci(const IndexerArgs& a, int64_t r0, int64_t r1, cudaStream_t st) {
  switch (a.nI) {
    case 1: return launch_scores_t<T, 1, CI>(a, r0, r1, st);
    case 2: return launch_scores_t<T, 2, CI>(a, r0, r1, st);
    case 4: return launch_scores_t<T, 4, CI>(a, r0, r1, st);
    case 8: return launch_scores_t<T, 8, CI>(a, r0, r1, st);
    case 16: return launch_scores_t<T, 16, CI>(a, r0, r1, st);
    case 32: return launch_scores_t<T, 32, CI>(a, r0, r1, st);
    case 64: return launch_scores_t<T, 64, CI>(a, r0, r1, st);
    default: return cudaErrorNotSupported;
  }
}

template <typename T>
cudaError_t launch_scores(const IndexerArgs& a, int64_t r0, int64_t r1, cudaStream_t st) {
  switch (a.cI) {
    case 32: return launch_scores_ci<T, 32>(a, r0, r1, st);
    case 64: return launch_scores_ci<T, 64>(a, r0, r1, st);
    case 128: return launch_scores_ci<T, 128>(a, r0, r1, st);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace

// Fixed score scratch of dsv4_indexer_topk_noalloc: a file-scope device array, so that
// callers without an allocator still get the indexer.  Every device that loads the
// library holds these bytes until the process exits.  Calls share the array; nothing in
// it has to start at zero (each score row is written before it is read).
static __device__ __align__(256) float g_noalloc_scores[kNoAllocScoreFloats];

cudaError_t noalloc_scores_scratch(float** ptr) {
  static std::mutex mu;
  static float* by_device[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!by_device[dev]) {
    // Host code sees g_noalloc_scores only as a stand-in symbol; the device address of this
    // device's copy comes from the runtime, with this device current.
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scores);
    if (e != cudaSuccess) return e;
    by_device[dev] = static_cast<float*>(p);
  }
  *ptr = by_device[dev];
  return cudaSuccess;
}

int64_t indexer_rows_per_chunk(int64_t total_rows, int P_cap, size_t bytes) {
  const int64_t per_row = (int64_t)P_cap * (int64_t)sizeof(float);
  int64_t r = per_row > 0 ? (int64_t)(bytes / per_row) : total_rows;
  if (r > total_rows) r = total_rows;
  if (r > 65535) r = 65535;  // the score grid's y extent is rows / (64 / nI) <= 65535
  return r;
}

cudaError_t launch_indexer_scores(const IndexerArgs& a, int dtype, int64_t r0, int64_t r1, cudaStream_t st) {
  return indexer_tc_supported(a, dtype) ? launch_indexer_tc_scores(a, r0, r1, st)
         : dtype == DSV4_BF16           ? launch_scores<__nv_bfloat16>(a, r0, r1, st)
                                        : launch_scores<float>(a, r0, r1, st);
}

cudaError_t launch_topk(const IndexerArgs& a, int64_t r0, int64_t r1, cudaStream_t st) {
  // Long rows and few of them (decode): 1024 threads per row, keys cached in shared memory.
  // Short rows, or long rows in their thousands (prefill): 256 threads per row, so that several
  // rows share an SM; long rows then re-read their keys from the score rows (in L2) instead of
  // caching them (measured on B200, DSA prefill, 32768 rows of up to 32768 scores: 3.14 ->
  // 2.83 ms; 64 decode rows: 29 -> 91 us, hence the row count).
  const int64_t rows = r1 - r0;
  const bool wide = a.P_cap > 4096 && rows < 4 * 148;
  const bool uncached = a.P_cap > 4096 && !wide;
  const size_t smem = uncached ? (size_t)kTopkListBytes
                               : (size_t)(a.P_cap < kTopkSmemKeys ? a.P_cap : kTopkSmemKeys) * sizeof(uint32_t);
  const int cache_keys = uncached ? 0 : (int)(smem / sizeof(uint32_t));
  void (*kern)(IndexerArgs, int64_t, int) = wide ? topk_kernel<1024> : topk_kernel<256>;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)(r1 - r0), wide ? 1024 : 256, smem, st>>>(a, r0, cache_keys);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_indexer_topk(const IndexerArgs& a, int dtype, cudaStream_t st) {
  const int64_t rows = (int64_t)a.B * a.Sq;
  for (int64_t r0 = 0; r0 < rows; r0 += a.rows_per_chunk) {
    const int64_t r1 = r0 + a.rows_per_chunk < rows ? r0 + a.rows_per_chunk : rows;
    if (indexer_tc_supported(a, dtype)) {
      // one query per sequence (decode): scores and top-k in one kernel when it applies
      const cudaError_t f = launch_indexer_tc_select(a, r0, r1, a.scores_cap, st);
      if (f == cudaSuccess) continue;
      if (f != cudaErrorNotSupported) return f;
    }
    cudaError_t e = launch_indexer_scores(a, dtype, r0, r1, st);
    if (e != cudaSuccess) return e;
    e = launch_topk(a, r0, r1, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace dsv4
