// Radix top-k selection over order-preserving 32-bit keys of fp32 scores, for one CTA-wide
// group of threads with its own barrier.
//
// Method: "DeepSeek-V4" doc, "Hybrid attention (§2.3)" CSA item — keep the index_topk
// highest-scoring entries per query (eq. 17); the tie rule of this build: among equal
// scores the lower entry index wins; -0 and +0 are equal.
//
// select_topk finds the K-th largest key T of keys key_of(0..n-1) by a 12-bit digit
// histogram followed by 12 and 8 more bits over the keys still matching the prefix (stopping
// early once the threshold digit holds exactly the keys still needed), then writes every
// index with a key above T and the `need` lowest indices with a key equal to T, in ascending
// index order: emit(slot, i) for slot = 0 .. K-1.
#pragma once

#include <stdint.h>

namespace dsv4 {

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0u) u = 0u;  // -0 and +0 are the same score
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kSelBins = 4096;  // radix digits of 12 bits

template <int NT>
struct SelShared {
  int wsum[NT / 32];
  int wcnt_gt[NT / 32], wcnt_eq[NT / 32];
  int bin, rest, cnt;
  uint32_t kmin, kmax;
};

// The digit holding the need-th largest key of a histogram (digits scanned from the top):
// sh->bin = that digit, sh->rest = how many keys of it are still needed, sh->cnt = its count.
// Thread t (t < NT) owns the descending run of digits [top - BPT + 1, top].
template <int NT, typename Sync>
__device__ __forceinline__ void select_digit(const uint32_t* hist, int need, int t, SelShared<NT>* sh, Sync sync) {
  constexpr int BPT = kSelBins / NT;
  const int lane = t & 31, warp = t >> 5;
  const int top = kSelBins - 1 - t * BPT;
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
  if (lane == 31) sh->wsum[warp] = incl;
  sync();
  if (warp == 0) {
    int v = lane < NT / 32 ? sh->wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += n;
    }
    if (lane < NT / 32) sh->wsum[lane] = v;
  }
  sync();
  incl += warp > 0 ? sh->wsum[warp - 1] : 0;
  const int excl = incl - sum;
  if (excl < need && need <= incl) {
    int run = excl;
#pragma unroll
    for (int k = 0; k < BPT; ++k) {
      if (run < need && need <= run + cnt[k]) {
        sh->bin = top - k;
        sh->rest = need - run;
        sh->cnt = cnt[k];
      }
      run += cnt[k];
    }
  }
  sync();
}

// Top-K of n > K keys (see the file comment).  t = this thread's rank in the group [0, NT);
// hist = kSelBins words of shared memory; every thread of the group calls it.  The digits are
// taken from rel = key - (smallest key), starting at the highest bit in which the keys differ:
// scores that share their sign and exponent (the candidates of a merge always do) would
// otherwise fall into a handful of bins, and the histogram's atomics would serialise on them.
template <int NT, typename KeyOf, typename Emit, typename Sync>
__device__ __forceinline__ void select_topk(int n, int K, int t, KeyOf key_of, Emit emit, uint32_t* hist,
                                            SelShared<NT>* sh, Sync sync) {
  constexpr int kWarps = NT / 32;
  const int lane = t & 31, warp = t >> 5;
  if (t == 0) {
    sh->kmin = 0xFFFFFFFFu;
    sh->kmax = 0u;
  }
  sync();
  uint32_t lmin = 0xFFFFFFFFu, lmax = 0u;
  for (int i0 = 0; i0 < n; i0 += 8 * NT) {
    uint32_t k[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * NT + t;
      k[u] = i < n ? key_of(i) : key_of(0);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      lmin = min(lmin, k[u]);
      lmax = max(lmax, k[u]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    lmin = min(lmin, __shfl_xor_sync(0xffffffffu, lmin, o));
    lmax = max(lmax, __shfl_xor_sync(0xffffffffu, lmax, o));
  }
  if (lane == 0) {
    atomicMin(&sh->kmin, lmin);
    atomicMax(&sh->kmax, lmax);
  }
  sync();
  const uint32_t k0 = sh->kmin;
  const uint32_t range = sh->kmax - k0;
  int lo = range ? 32 - __clz(range) : 0;  // bits of rel still to resolve: [0, lo)
  uint32_t prefix = 0u, mask = 0u;
  int need = K, cnt = -1;
  while (lo > 0 && cnt != need) {
    const int dlo = lo > 12 ? lo - 12 : 0;
    const uint32_t dmask = (1u << (lo - dlo)) - 1u;
    for (int i = t; i < kSelBins; i += NT) hist[i] = 0u;
    sync();
    for (int i0 = 0; i0 < n; i0 += 8 * NT) {  // eight keys read before any is counted
      uint32_t r[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * NT + t;
        r[u] = i < n ? key_of(i) - k0 : 0u;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * NT + t;
        if (i < n && (r[u] & mask) == prefix) atomicAdd(&hist[(r[u] >> dlo) & dmask], 1u);
      }
    }
    sync();
    select_digit<NT>(hist, need, t, sh, sync);
    prefix |= (uint32_t)sh->bin << dlo;
    mask |= dmask << dlo;
    need = sh->rest;
    cnt = sh->cnt;
    lo = dlo;
  }
  // ordered compaction: each warp owns a contiguous segment of the keys; per-warp counts,
  // a scan over warps, then ordered writes
  const int seg = (n + kWarps - 1) / kWarps;
  const int s_lo = min(n, warp * seg), s_hi = min(n, s_lo + seg);
  int n_gt = 0, n_eq = 0;
  for (int i = s_lo + lane; i < s_hi; i += 32) {
    const uint32_t k = (key_of(i) - k0) & mask;
    n_gt += k > prefix;
    n_eq += k == prefix;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    n_gt += __shfl_xor_sync(0xffffffffu, n_gt, o);
    n_eq += __shfl_xor_sync(0xffffffffu, n_eq, o);
  }
  if (lane == 0) {
    sh->wcnt_gt[warp] = n_gt;
    sh->wcnt_eq[warp] = n_eq;
  }
  sync();
  int pos_gt = 0, pos_eq = 0;
  for (int w = 0; w < warp; ++w) {
    pos_gt += sh->wcnt_gt[w];
    pos_eq += sh->wcnt_eq[w];
  }
  for (int base = s_lo; base < s_hi; base += 32) {
    const int i = base + lane;
    const uint32_t k = i < s_hi ? (key_of(i) - k0) & mask : 0u;
    const bool gt = i < s_hi && k > prefix;
    const bool eq = i < s_hi && k == prefix;
    const unsigned bgt = __ballot_sync(0xffffffffu, gt), beq = __ballot_sync(0xffffffffu, eq);
    const unsigned below = (1u << lane) - 1u;
    const int my_eq_rank = pos_eq + __popc(beq & below);
    const int slot = pos_gt + __popc(bgt & below) + min(my_eq_rank, need);
    if ((gt || (eq && my_eq_rank < need)) && slot < K) emit(slot, i);
    pos_gt += __popc(bgt);
    pos_eq += __popc(beq);
  }
  sync();
}

}  // namespace dsv4
