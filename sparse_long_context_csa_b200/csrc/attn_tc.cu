// Sparse shared-K=V MQA attention with sink on the sm_100a tensor cores (tcgen05 + TMEM),
// bf16 inputs, fp32 accumulation.
//
// Method: "DeepSeek-V4" doc, "Hybrid attention (§2.3)" — one K=V head read as both key and
// value, partial interleaved RoPE with the -i rotation of the output rope slice (eq. 26),
// per-head sink (eq. 27), the sliding-window K=V rows concatenated with the compressor
// entries picked by the Lightning Indexer; "DeepSeek-V3.2" doc, DSA item 2 (attention over
// the selected tokens only).
//
// Design.  A persistent CTA per SM walks its queries; the 64 heads of a query share every
// key row (MQA).
//  * Keys of a query = window rows, then the selected pool entries, cut into 128-key tiles.
//    The eight softmax warps copy a tile themselves, chunk by chunk (64 channels), with
//    16-byte cp.async copies straight into the 128B-swizzled operand layout, right after
//    handing the previous tile's probabilities to the MMA: the copies overlap PV.  (Measured
//    on B200: random 128-byte row pieces move at ~18 B/clk per SM from 2 issuing warps and
//    ~55 B/clk from 8; TMA tile::gather4 ran at ~7 B/clk, and 128-row TMA boxes of window
//    rows were slower than cp.async as well.)  Every chunk has its own "full" barrier, so
//    S^T starts on the first chunk that lands; the whole tile is released by one barrier
//    committed after its PV products (a tcgen05.commit between MMA groups holds up the
//    issuing thread, so PV is issued as one uninterrupted run of MMAs).
//  * Scores are computed transposed, S^T[key, head] = K_tile . Q^T (M = 128 keys keeps the
//    tensor core at full rate; 64 heads alone would be a half-rate M=64 shape), and the same
//    shared-memory tile is read again as V^T (MN-major) for O^T[dim, head] += V^T . P^T: K=V
//    costs one gather for both products.
//  * q (64 heads x D) arrives by one TMA burst in the same swizzled layout as soon as the
//    previous query's last S^T has read the buffer; a prep warp scans the query's index row,
//    then rotates q's rope slice in place while the previous query finishes.
//  * Eight softmax warps, two per TMEM lane quadrant: a thread owns one key and 32 heads (two
//    warps per SM sub-partition hide each other's latencies; measured: splitting the MMAs
//    into N = 32 halves to overlap them with the softmax was slower than N = 64).  The running
//    max per head starts at the sink logit and is raised only when a score exceeds it by
//    more than 2^8 (the O^T columns are then rescaled in TMEM), so a typical tile needs no
//    cross-thread reduction.
//  * Few queries (decode): each query's tiles are split over several CTAs, which write
//    unnormalised partial outputs and softmax statistics to the workspace; a small combine
//    kernel adds the sink, normalises and rotates.
//  * TMEM: S^T 64 columns, O^T dv/128 tiles x 64 columns.  The epilogue reads O^T (lane =
//    channel), swaps half of its heads with the neighbouring lane so that each lane holds
//    channel pairs (d, d+1), applies 1/denominator and the -qpos rotation and stores pairs.
// Warp roles: 0 query prep (descriptor, q load, RoPE of q), 1 MMA issuer + TMEM owner,
//             2-9 key copies + softmax/epilogue (heads 0-31: warps 2-5, 32-63: warps 6-9).
// Every wait is bounded; a role that gives up records g_attn_tc_error and all roles leave
// their loops together (warp votes / barrier reductions), free TMEM and return.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"
#include "tc_ptx.cuh"

namespace dsv4 {

__device__ int g_attn_tc_error = 0;  // non-zero: a pipeline wait gave up (the CTA stopped early)

namespace {

constexpr int kH = 64;
constexpr int kHalf = 32;      // heads per softmax half
constexpr int kTile = 128;
constexpr int kThreads = 320;  // 10 warps
constexpr int kMaxChunks = 9;  // D <= 576
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: p <= 2^8 between rescales
constexpr uint32_t kWaitLimit = 1u << 20;  // mbarrier polls before a wait gives up
constexpr int kSelKeys = 2048;  // selection inside the kernel: score rows of at most this many entries
constexpr int kSelK = 512;      // ... and index lists of at most this many slots
constexpr uint32_t kMiscBytes = 8192;

struct TcParams {
  AttnArgs a;
  double inv_freq[64];  // theta^(-2k/R), k < R/2
  int64_t nrows;        // B * Sq queries
  int64_t nitems;       // work items = queries x key splits
  int tma_win;          // the window rows are a plain [B, kv_rows, D] tensor: map_win covers it
  int tma_pool;         // every visible pool entry is a key (no index lists): map_pool covers the pool
};

struct Smem {
  uint32_t q, k, p, misc, total;
};

__host__ __device__ inline Smem smem_layout(int D) {
  const int nch = D / 64;
  Smem s;
  s.q = 0;
  s.k = s.q + nch * 8192;
  const bool alias = D > 512;  // P^T reuses the last K chunk (those channels are not values)
  s.p = alias ? s.k + (nch - 1) * 16384 : s.k + nch * 16384;
  s.misc = alias ? s.k + nch * 16384 : s.p + 16384;
  s.total = s.misc + kMiscBytes;
  return s;
}

struct QDesc {
  int64_t qrow, item;
  int t, vis, wlo, nw, nw4, npool, ntiles, tile0;  // this item's tiles: [tile0, tile0 + ntiles)
  float cs[64], sn[64];  // RoPE table at the query position
  int16_t sidx[kSelK];   // the query's index list when the kernel selects it from a score row
};

struct Misc {
  uint64_t cfull[kMaxChunks];
  uint64_t qfull, qready, qfree, sfull, pfull;
  uint64_t odone;  // PV of a tile done: O^T is current and the key tile may be overwritten
  uint64_t dfull[2], dfree[2];
  uint32_t tmem_base;
  int abort_flag;
  int rescale_cnt[2][2];
  float m[kH];
  float fac[kH];
  float red[4][kH];
  float inv_l[kH];
  uint32_t sel_hist[256];  // radix histogram of the prep warp's selection
  QDesc desc[2];
};
static_assert(sizeof(Misc) <= kMiscBytes, "misc block exceeds its reservation");

__device__ __forceinline__ bool wait_ok(uint64_t* bar, uint32_t parity) {
  return tc::mbar_wait(bar, parity, kWaitLimit);
}

// One warp's top-K of the n scores sc[0..n), n <= kSelKeys, K <= kSelK: the same list as
// dsv4_topk_select ("DeepSeek-V4" doc, Hybrid attention (§2.3), CSA item, eq. 17: the
// index_topk highest-scoring entries; among equal scores the lower entry wins, -0 equals +0):
// the kept entries in ascending order in sidx[0..min(K, n)), then -1 up to K.  Lane l keeps
// the order keys of entries l + 32j in registers; the threshold key is found by 8-bit radix
// digits of (key - smallest key), from the highest bit in which the keys differ, over a
// 256-bin shared histogram; the ordered output is one pass of ballots in entry order.
__device__ __forceinline__ void warp_select(const float* __restrict__ sc, int n, int K, int16_t* sidx,
                                         uint32_t* hist) {
  const int lane = threadIdx.x & 31;
  if (n <= K) {
    for (int j = lane; j < K; j += 32) sidx[j] = (int16_t)(j < n ? j : -1);
    __syncwarp();
    return;
  }
  constexpr int kPer = kSelKeys / 32;
  uint32_t key[kPer];
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int i = lane + 32 * j;
    key[j] = i < n ? order_key(sc[i]) : 0u;
  }
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    if (lane + 32 * j < n) {
      kmin = min(kmin, key[j]);
      kmax = max(kmax, key[j]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  const uint32_t range = kmax - kmin;
  int lo = range ? 32 - __clz(range) : 0;  // bits of (key - kmin) still to resolve: [0, lo)
  uint32_t prefix = 0u, mask = 0u;
  int need = K, cnt = -1;
  while (lo > 0 && cnt != need) {
    const int dlo = lo > 8 ? lo - 8 : 0;
    const uint32_t dmask = (1u << (lo - dlo)) - 1u;
#pragma unroll
    for (int b = 0; b < 8; ++b) hist[lane + 32 * b] = 0u;
    __syncwarp();
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const uint32_t r = key[j] - kmin;
      if (lane + 32 * j < n && (r & mask) == prefix) atomicAdd(&hist[(r >> dlo) & dmask], 1u);
    }
    __syncwarp();
    // bins from the top: lane l owns bins 255 - 8l .. 248 - 8l
    int c8[8], sum = 0;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      c8[b] = (int)hist[255 - 8 * lane - b];
      sum += c8[b];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const int excl = incl - sum;
    int bin = -1, rest = 0, bc = 0;
    if (excl < need && need <= incl) {
      int run = excl;
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        if (bin < 0 && need <= run + c8[b]) {
          bin = 255 - 8 * lane - b;
          rest = need - run;
          bc = c8[b];
        }
        run += c8[b];
      }
    }
    const int src = __ffs(__ballot_sync(0xffffffffu, bin >= 0)) - 1;
    bin = __shfl_sync(0xffffffffu, bin, src);
    rest = __shfl_sync(0xffffffffu, rest, src);
    bc = __shfl_sync(0xffffffffu, bc, src);
    prefix |= (uint32_t)bin << dlo;
    mask |= dmask << dlo;
    need = rest;
    cnt = bc;
    lo = dlo;
    __syncwarp();
  }
  // every entry above the prefix, and the `need` lowest-index entries equal to it
  int pos_gt = 0, pos_eq = 0;
  const unsigned below = (1u << lane) - 1u;
#pragma unroll
  for (int j = 0; j < kPer; ++j) {
    const int i = lane + 32 * j;
    const uint32_t r = (key[j] - kmin) & mask;
    const bool gt = i < n && r > prefix, eq = i < n && r == prefix;
    const unsigned bgt = __ballot_sync(0xffffffffu, gt), beq = __ballot_sync(0xffffffffu, eq);
    const int my_eq = pos_eq + __popc(beq & below);
    const int slot = pos_gt + __popc(bgt & below) + min(my_eq, need);
    if (gt || (eq && my_eq < need)) sidx[slot] = (int16_t)i;
    pos_gt += __popc(bgt);
    pos_eq += __popc(beq);
  }
  __syncwarp();
}

// kSel: the index lists are selected here from score rows (a.scores); the other
// instantiation carries none of that code.
template <bool kSel>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_win,
                   const __grid_constant__ CUtensorMap map_pool, const __grid_constant__ TcParams P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const AttnArgs& a = P.a;
  const int D = a.D;
  const int nch = D / 64;
  const int nvt = a.dv / 128;
  const Smem L = smem_layout(D);
  Misc* ms = reinterpret_cast<Misc*>(smem + L.misc);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if ((tc::smem_u32(smem) & 1023u) != 0) {  // the swizzle atoms need a 1024-byte aligned base
    if (tid == 0) atomicExch(&g_attn_tc_error, 3);
    return;
  }
  const int64_t nq_cta = P.nitems > (int64_t)blockIdx.x ? (P.nitems - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  if (tid == 0) {
    for (int c = 0; c < kMaxChunks; ++c) {
      tc::mbar_init(&ms->cfull[c], 256);  // one cp.async arrival per softmax thread
    }
    tc::mbar_init(&ms->qfull, 1);
    tc::mbar_init(&ms->qready, 32);
    tc::mbar_init(&ms->qfree, 1);
    tc::mbar_init(&ms->odone, 1);
    tc::mbar_init(&ms->sfull, 1);
    tc::mbar_init(&ms->pfull, 256);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&ms->dfull[i], 32);
      tc::mbar_init(&ms->dfree[i], 3);  // MMA and the two softmax halves
    }
    for (int i = 0; i < 4; ++i) (&ms->rescale_cnt[0][0])[i] = 0;
    ms->abort_flag = 0;
    tc::mbar_fence_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&ms->tmem_base, 512);
    tc::tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tensormap(&map_q);
    if (P.tma_win) tc::prefetch_tensormap(&map_win);
    if (P.tma_pool) tc::prefetch_tensormap(&map_pool);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = ms->tmem_base;
  const uint32_t tS = tmem, tO = tmem + 64;

  if (warp == 0) {
    // ================================================================ query prep (1 warp)
    const int R = a.R;
    const int rope_lo = D - R;
    bool ok = true;
    for (int64_t n = 0; n < nq_cta; ++n) {
      const int slot = (int)(n & 1);
      const int64_t item = blockIdx.x + n * gridDim.x;
      const int64_t qrow = item / a.nsplit;
      const int split = (int)(item % a.nsplit);
      if (n >= 2 && !__all_sync(0xffffffffu, wait_ok(&ms->dfree[slot], ((n >> 1) - 1) & 1))) {
        ok = false;
        break;
      }
      QDesc* d = &ms->desc[slot];
      const int s = (int)(qrow % a.Sq);
      const int t = query_cache_index(a.q_index, qrow, s);
      const int vis = visible_entries(t, a.m, a.P_cap);
      const int wlo = t - a.n_win + 1 > 0 ? t - a.n_win + 1 : 0;
      int nw = a.n_win > 0 ? t - wlo + 1 : 0;
      if (nw < 0) nw = 0;
      if (!a.win_ring && wlo + nw > a.kv_rows) nw = a.kv_rows > wlo ? a.kv_rows - wlo : 0;
      // last valid slot of the index row (slots past it are skipped, holes are masked)
      int last = 0;
      if (kSel) {
        // select the index list from the score row (entries w < vis)
        warp_select(a.scores + qrow * a.P_cap, vis, a.topk, d->sidx, ms->sel_hist);
        last = min(a.topk, vis);
        if (a.idx_out)
          for (int k = lane; k < a.topk; k += 32) a.idx_out[qrow * a.topk + k] = d->sidx[k];
      } else if (a.idx) {
        const int32_t* ir = a.idx + qrow * a.topk;
        for (int k = lane; k < a.topk; k += 32) {
          const int w = ir[k];
          if (w >= 0 && w < vis) last = k + 1;
        }
        for (int o = 16; o > 0; o >>= 1) last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
      } else {
        last = vis > 0 ? vis : 0;
      }
      if (a.rope_q || a.rotate_out) {
        for (int k = lane; k < R / 2; k += 32) {
          double ang = (double)a.qpos[qrow] * P.inv_freq[k];
          ang -= rint(ang * 0.15915494309189535) * 6.283185307179586;  // reduce to [-pi, pi]
          float c, sn;
          sincosf((float)ang, &sn, &c);
          d->cs[k] = c;
          d->sn[k] = sn;
        }
      }
      if (lane == 0) {
        d->qrow = qrow;
        d->item = item;
        d->t = t;
        d->vis = vis;
        d->wlo = wlo;
        d->nw = nw;
        d->nw4 = (nw + 3) & ~3;
        d->npool = last;
        const int NK = d->nw4 + last;
        const int nt_all = (NK + kTile - 1) / kTile;
        const int per = (nt_all + a.nsplit - 1) / a.nsplit;
        const int lo = min(nt_all, split * per);
        d->tile0 = lo;
        d->ntiles = min(nt_all, lo + per) - lo;
      }
      __syncwarp();
      tc::mbar_arrive(&ms->dfull[slot]);
      // q of this query, once the previous query's last S^T has read the buffer
      if (n > 0 && !__all_sync(0xffffffffu, wait_ok(&ms->qfree, (n - 1) & 1))) {
        ok = false;
        break;
      }
      if (lane == 0) {
        tc::mbar_arrive_expect_tx(&ms->qfull, (uint32_t)(kH * D * 2));
        for (int c = 0; c < nch; ++c)
          tc::tma_load_2d(smem + L.q + c * 8192, &map_q, c * 64, (int)(qrow * kH), &ms->qfull);
      }
      if (!__all_sync(0xffffffffu, wait_ok(&ms->qfull, n & 1))) {
        ok = false;
        break;
      }
      // rotate the rope slice of q in place: lane owns pair k, 8 heads per batch
      if (a.rope_q) {
        for (int k = lane; k < R / 2; k += 32) {
          const float c = d->cs[k], sn = d->sn[k];
          const int dd = rope_lo + 2 * k;
          const uint32_t col = (dd / 64) * 8192 + (dd % 8) * 2;
          const int unit = (dd % 64) / 8;
          for (int h0 = 0; h0 < kH; h0 += 8) {
            __nv_bfloat162 v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int h = h0 + e;
              v[e] = *reinterpret_cast<const __nv_bfloat162*>(smem + L.q + col + h * 128 + ((unit ^ (h & 7)) * 16));
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int h = h0 + e;
              const float2 f = __bfloat1622float2(v[e]);
              *reinterpret_cast<__nv_bfloat162*>(smem + L.q + col + h * 128 + ((unit ^ (h & 7)) * 16)) =
                  __floats2bfloat162_rn(f.x * c - f.y * sn, f.x * sn + f.y * c);
            }
          }
        }
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&ms->qready);
    }
    if (!ok && lane == 0) atomicExch(&g_attn_tc_error, 6);
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    // Per tile: S^T for heads 0-31, S^T for heads 32-63, PV for heads 0-31, PV for 32-63, so
    // the tensor core works on one half while the softmax of the other half runs.
    const uint32_t idS = tc::idesc_bf16_f32(128, 64, 0, 0);
    const uint32_t idO = tc::idesc_bf16_f32(128, 64, 1, 1);
    const uint32_t kbase = tc::smem_u32(smem + L.k);
    const uint32_t qbase = tc::smem_u32(smem + L.q);
    const uint32_t pbase = tc::smem_u32(smem + L.p);
    // Descriptors differ between MMAs only in their start address (bits 0-13, in 16-byte
    // units), so each is formed once and stepped by adding the offset.
    const uint64_t dK = tc::sdesc_sw128(kbase, 16, 1024);        // K tile, K-major (S^T A)
    const uint64_t dQ = tc::sdesc_sw128(qbase, 16, 1024);        // q, K-major (S^T B)
    const uint64_t dV = tc::sdesc_sw128(kbase, 16384, 1024);     // K tile, MN-major (PV A)
    const uint64_t dP = tc::sdesc_sw128(pbase, 16384, 1024);     // P^T, MN-major (PV B)
    uint32_t g = 0;
    bool ok = true;
    for (int64_t n = 0; n < nq_cta && ok; ++n) {
      const int slot = (int)(n & 1);
      if (!__all_sync(0xffffffffu, wait_ok(&ms->dfull[slot], (n >> 1) & 1))) {
        ok = false;
        break;
      }
      const QDesc* d = &ms->desc[slot];
      const int ntiles = d->ntiles;
      const int NK = d->nw4 + d->npool;
      const int tile0 = d->tile0;
      if (!__all_sync(0xffffffffu, wait_ok(&ms->qready, n & 1))) {
        ok = false;
        break;
      }
      for (int i = 0; i < ntiles; ++i, ++g) {
        // S^T (heads 0-31) chunk by chunk as the copies land
        for (int c = 0; c < nch; ++c) {
          if (!__all_sync(0xffffffffu, wait_ok(&ms->cfull[c], g & 1))) {
            ok = false;
            break;
          }
          tc::fence_proxy_async_smem();  // cp.async wrote the chunk through the generic proxy
          tc::tc_fence_after();
          if (lane == 0) {
            const uint64_t ac = dK + (uint64_t)(c * 1024), bc = dQ + (uint64_t)(c * 512);
#pragma unroll
            for (int kq = 0; kq < 4; ++kq)
              tc::umma_f16(tS, ac + 2 * kq, bc + 2 * kq, idS, (c > 0 || kq > 0) ? 1u : 0u);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (lane == 0) {
          tc::umma_commit(&ms->sfull);
          if (i == ntiles - 1) tc::umma_commit(&ms->qfree);
        }
        __syncwarp();
        const int nvalid = min(kTile, NK - (tile0 + i) * kTile);
        const int nsteps = (nvalid + 15) / 16;
        {
          if (!__all_sync(0xffffffffu, wait_ok(&ms->pfull, g & 1))) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          if (lane == 0) {
            for (int j = 0; j < nvt; ++j) {
              const uint64_t aj = dV + (uint64_t)(j * 2048);
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)
                if (kk < nsteps) tc::umma_f16(tO + 64 * j, aj + 128 * kk, dP + 128 * kk, idO, (i > 0 || kk > 0) ? 1u : 0u);
            }
            tc::umma_commit(&ms->odone);
          }
          __syncwarp();
        }
        if (!ok) break;
      }
      if (!ok) break;
      if (ntiles == 0 && lane == 0) tc::umma_commit(&ms->qfree);  // q was never read
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&ms->dfree[slot]);
    }
    if (!ok && lane == 0) atomicExch(&g_attn_tc_error, 2);
  } else {
    // ================================================================ copies + softmax / epilogue
    // Two halves of 4 warps: half hh owns heads [32hh, 32hh+32); thread = key (TMEM lane).
    // The 256 threads also copy the key tiles, one tile ahead: right after handing tile i's
    // probabilities to the MMA they issue the copies of the next tile (possibly the first
    // tile of the next query), so the copies overlap PV(i) and the epilogue.
    const int hh = (warp - 2) >> 2;
    const int q4 = warp & 3;                  // TMEM lane quadrant of this warp
    const int kk = q4 * 32 + lane;            // key of the tile owned by this thread
    const int st = tid - 64 - 128 * hh;       // 0..127 within the half
    const int ct = tid - 64;                  // 0..255 over both halves (copy lanes)
    const int bar_id = 1 + hh;
    const int h0 = kHalf * hh;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const float c1 = a.scale * kLog2e;

    // Copy key tile i of query descriptor d as tile number gcopy of this CTA.  Threads wait on
    // the chunk barriers on their own; a give-up sets abort_flag, checked at the next barrier.
    auto copy_tile = [&](const QDesc* d, int i, uint32_t gcopy) {
      const int64_t qrow = d->qrow;
      const int b = (int)(qrow / a.Sq);
      const __nv_bfloat16* win_base =
          static_cast<const __nv_bfloat16*>(a.kv_win) + (int64_t)b * (a.win_ring ? a.win_ring : a.kv_rows) * D;
      const __nv_bfloat16* pool_base = static_cast<const __nv_bfloat16*>(a.pool) + (int64_t)b * a.P_cap * D;
      // index list: selected in this kernel (shared memory) or given (global)
      const int16_t* irs = kSel ? d->sidx : nullptr;
      const int32_t* ir = a.idx ? a.idx + qrow * a.topk : nullptr;
      const int nw = d->nw, nw4 = d->nw4, npool = d->npool, vis = d->vis, wlo = d->wlo;
      const int cu = ct & 7;
      const int k0 = (d->tile0 + i) * kTile;
      const int nvalid = min(kTile, nw4 + npool - k0);
      const int nk = (nvalid + 15) & ~15;
      // A tile whose keys are all window rows, or all pool entries taken in order (no index
      // list), is one run of 128 consecutive rows: TMA boxes of 64 channels x 128 rows land it
      // in the same 128B-swizzled layout (rows past the keys are masked; rows past the
      // tensor's end read zeros).
      const bool all_win = k0 + kTile <= nw4 || npool == 0;
      const bool all_pool = k0 >= nw4;
      const CUtensorMap* tmap = nullptr;
      int row0 = 0;
      if (all_win && P.tma_win) {
        tmap = &map_win;
        row0 = b * a.kv_rows + wlo + k0;
      } else if (all_pool && P.tma_pool) {
        tmap = &map_pool;
        row0 = b * a.P_cap + (k0 - nw4);
      }
      if (tmap) {
        if (gcopy > 0 && !wait_ok(&ms->odone, (gcopy - 1) & 1)) ms->abort_flag = 1;
        for (int c = 0; c < nch; ++c) {
          if (ct == 0) {
            tc::mbar_arrive_expect_tx(&ms->cfull[c], 16384u);
            tc::tma_load_2d(smem + L.k + c * 16384, tmap, c * 64, row0, &ms->cfull[c]);
          } else {
            tc::mbar_arrive(&ms->cfull[c]);
          }
        }
        return;
      }
      const __nv_bfloat16* src[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = (ct >> 3) + 32 * j;
        const int kr = k0 + r;
        if (kr >= nw4 && npool > 0) {
          const int p = kr - nw4;
          const int w = p < npool ? (irs ? (int)irs[p] : ir ? ir[p] : p) : -1;
          src[j] = pool_base + (int64_t)((w >= 0 && w < vis) ? w : 0) * D + cu * 8;
        } else {
          const int jj = kr < nw ? wlo + kr : wlo;
          src[j] = win_base + (int64_t)(a.win_ring ? jj % a.win_ring : jj) * D + cu * 8;
        }
      }
      if (gcopy > 0 && !wait_ok(&ms->odone, (gcopy - 1) & 1)) ms->abort_flag = 1;
      for (int c = 0; c < nch; ++c) {
        uint8_t* cb = smem + L.k + c * 16384;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = (ct >> 3) + 32 * j;
          if (r < nk) tc::cp_async_16(cb + r * 128 + ((cu ^ (r & 7)) * 16), src[j] + c * 64);
        }
        tc::cp_async_arrive_noinc(&ms->cfull[c]);
      }
    };

    uint32_t g = 0;         // tiles softmaxed so far (all queries of this CTA)
    bool first_copied = false;  // tile 0 of the current query was copied at the end of the previous one
    bool ok = true;
    for (int64_t n = 0; n < nq_cta && ok; ++n) {
      const int slot = (int)(n & 1);
      ok = tc::named_bar_and(bar_id, 128, wait_ok(&ms->dfull[slot], (n >> 1) & 1));
      if (!ok) break;
      const QDesc* d = &ms->desc[slot];
      const int64_t qrow = d->qrow;
      const int ntiles = d->ntiles, nw = d->nw, nw4 = d->nw4, npool = d->npool, vis = d->vis;
      const int16_t* irs = kSel ? d->sidx : nullptr;
      const int32_t* ir = a.idx ? a.idx + qrow * a.topk : nullptr;
      if (!first_copied && ntiles > 0) copy_tile(d, 0, g);
      first_copied = false;
      if (st < kHalf) ms->m[h0 + st] = a.sink[h0 + st] * kLog2e;
      tc::named_bar_sync(bar_id, 128);
      float l[kHalf];
#pragma unroll
      for (int h = 0; h < kHalf; ++h) l[h] = 0.f;
      for (int i = 0; i < ntiles; ++i, ++g) {
        // validity of this thread's key (the index read is issued before the wait)
        const int k = (d->tile0 + i) * kTile + kk;
        bool valid;
        if (k < nw4) {
          valid = k < nw;
        } else {
          const int p = k - nw4;
          if (p < npool) {
            const int w = irs ? (int)irs[p] : ir ? ir[p] : p;
            valid = w >= 0 && w < vis;
          } else {
            valid = false;
          }
        }
        ok = tc::named_bar_and(bar_id, 128, wait_ok(&ms->sfull, g & 1) && ms->abort_flag == 0);
        if (!ok) break;
        tc::tc_fence_after();
        float sv[kHalf];
        tc::tmem_ld_x32(tS + h0 + lane_off, sv);
        const float* mr = ms->m + h0;  // running max of this half (shared-memory broadcast reads)
        bool need = false;
#pragma unroll
        for (int h = 0; h < kHalf; ++h) {
          sv[h] *= c1;
          need |= valid && (sv[h] - mr[h] > kRescaleThreshold);
        }
        if (__any_sync(0xffffffffu, need) && lane == 0) atomicAdd(&ms->rescale_cnt[hh][g & 1], 1);
        tc::named_bar_sync(bar_id, 128);
        const bool rescale = ms->rescale_cnt[hh][g & 1] != 0;
        if (st == 0) ms->rescale_cnt[hh][(g + 1) & 1] = 0;
        if (rescale) {
#pragma unroll
          for (int h = 0; h < kHalf; ++h) {
            const float v = warp_max(valid ? sv[h] : -INFINITY);
            if (lane == 0) ms->red[q4][h0 + h] = v;
          }
          tc::named_bar_sync(bar_id, 128);
          if (st < kHalf) {
            const int h = h0 + st;
            const float tm = fmaxf(fmaxf(ms->red[0][h], ms->red[1][h]), fmaxf(ms->red[2][h], ms->red[3][h]));
            const float mo = ms->m[h];
            const float mn = fmaxf(mo, tm);
            ms->fac[h] = tc::ex2(mo - mn);
            ms->m[h] = mn;
          }
          tc::named_bar_sync(bar_id, 128);
#pragma unroll
          for (int h = 0; h < kHalf; ++h) l[h] *= ms->fac[h0 + h];
          if (i > 0) {  // O^T holds tiles 0..i-1; S^T(i) completing implies PV(i-1) completed
            float o[kHalf];
            for (int j = 0; j < nvt; ++j) {
              tc::tmem_ld_x32(tO + 64 * j + h0 + lane_off, o);
#pragma unroll
              for (int h = 0; h < kHalf; ++h) o[h] *= ms->fac[h0 + h];
              tc::tmem_st_x32(tO + 64 * j + h0 + lane_off, o);
            }
          }
          tc::named_bar_sync(bar_id, 128);
        }
        // probabilities -> this half of P^T row `kk` (bf16, 128B-swizzled MN-major B operand)
        uint8_t* prow = smem + L.p + kk * 128;
#pragma unroll
        for (int uu = 0; uu < 4; ++uu) {
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int h = uu * 8 + 2 * e;
            const float p0 = valid ? tc::ex2(sv[h] - mr[h]) : 0.f;
            const float p1 = valid ? tc::ex2(sv[h + 1] - mr[h + 1]) : 0.f;
            l[h] += p0;
            l[h + 1] += p1;
            __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
            w4[e] = *reinterpret_cast<uint32_t*>(&pr);
          }
          *reinterpret_cast<uint4*>(prow + (((4 * hh + uu) ^ (kk & 7)) * 16)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        tc::mbar_arrive(&ms->pfull);
        // copies of the next tile: this query's next tile, or the next query's first tile
        if (i + 1 < ntiles) {
          copy_tile(d, i + 1, g + 1);
        } else if (n + 1 < nq_cta) {
          const int ns = (int)((n + 1) & 1);
          ok = tc::named_bar_and(bar_id, 128, wait_ok(&ms->dfull[ns], ((n + 1) >> 1) & 1));
          if (!ok) break;
          if (ms->desc[ns].ntiles > 0) {
            copy_tile(&ms->desc[ns], 0, g + 1);
            first_copied = true;
          }
        }
      }
      if (!ok) break;

      // ---------------------------------------------------------- epilogue of query n
      // denominators: halving butterfly over the warp (each lane ends with one head sum),
      // then the 4 warps of the half meet in shared memory
      {
#pragma unroll
        for (int sft = 16, half = 16; sft >= 1; sft >>= 1, half >>= 1) {
          const bool up = (lane & sft) != 0;
#pragma unroll
          for (int h = 0; h < half; ++h) {
            const float keep = up ? l[h + half] : l[h];
            const float send = up ? l[h] : l[h + half];
            l[h] = keep + __shfl_xor_sync(0xffffffffu, send, sft);
          }
        }
        int hb = 0;
#pragma unroll
        for (int sft = 16, half = 16; sft >= 1; sft >>= 1, half >>= 1)
          if (lane & sft) hb += half;
        ms->red[q4][h0 + hb] = l[0];
      }
      const bool have = ntiles > 0;
      if (have) {
        ok = tc::named_bar_and(bar_id, 128, wait_ok(&ms->odone, (g - 1) & 1));
        if (!ok) break;
      } else {
        tc::named_bar_sync(bar_id, 128);
      }
      tc::tc_fence_after();
      if (a.nsplit > 1) {
        // split over keys: unnormalised O, running max (log2 units) and partial denominator of
        // this item; the combine kernel adds the sink, normalises and rotates.
        float* po = a.part + d->item * (int64_t)kH * (a.dv + 2);
        float* pml = po + (int64_t)kH * a.dv;
        if (st < kHalf) {
          const int h = h0 + st;
          pml[2 * h] = ms->m[h];
          pml[2 * h + 1] = ms->red[0][h] + ms->red[1][h] + ms->red[2][h] + ms->red[3][h];
        }
        const bool odd = (lane & 1) != 0;
        const int hl = h0 + (odd ? kHalf / 2 : 0);
        for (int j = 0; j < nvt; ++j) {
          float o[kHalf];
          if (have) {
            tc::tmem_ld_x32(tO + 64 * j + h0 + lane_off, o);
          } else {
#pragma unroll
            for (int h = 0; h < kHalf; ++h) o[h] = 0.f;
          }
          const int dd = 128 * j + q4 * 32 + (lane & ~1);
#pragma unroll
          for (int i = 0; i < kHalf / 2; ++i) {
            const float keep = odd ? o[i + kHalf / 2] : o[i];
            const float recv = __shfl_xor_sync(0xffffffffu, odd ? o[i] : o[i + kHalf / 2], 1);
            *reinterpret_cast<float2*>(po + (int64_t)(hl + i) * a.dv + dd) =
                odd ? make_float2(recv, keep) : make_float2(keep, recv);
          }
        }
        tc::tc_fence_before();
        tc::named_bar_sync(bar_id, 128);
        if (st == 0) tc::mbar_arrive(&ms->dfree[slot]);
        continue;
      }
      if (st < kHalf) {
        const int h = h0 + st;
        const float sum = ms->red[0][h] + ms->red[1][h] + ms->red[2][h] + ms->red[3][h];
        ms->inv_l[h] = 1.f / (sum + tc::ex2(a.sink[h] * kLog2e - ms->m[h]));
      }
      tc::named_bar_sync(bar_id, 128);
      // O^T lane = dim, column = head.  One exchange between neighbouring lanes (dims d, d+1)
      // leaves the even lane with both dims of heads 0-15 of the half and the odd lane with
      // both dims of heads 16-31: every store is one (d, d+1) pair (64 contiguous bytes of a
      // head across the 16 lanes), and the rope pairs sit in one lane for the -qpos rotation.
      const int rope_lo = D - a.R;
      const bool odd = (lane & 1) != 0;
      const int hl = h0 + (odd ? kHalf / 2 : 0);  // first head this lane stores
      __nv_bfloat16* og = static_cast<__nv_bfloat16*>(a.out) + qrow * kH * a.dv;
      float il[kHalf / 2];
#pragma unroll
      for (int i = 0; i < kHalf / 2; ++i) il[i] = ms->inv_l[hl + i];
      for (int j = 0; j < nvt; ++j) {
        float o[kHalf];
        if (have) {
          tc::tmem_ld_x32(tO + 64 * j + h0 + lane_off, o);
        } else {
#pragma unroll
          for (int h = 0; h < kHalf; ++h) o[h] = 0.f;
        }
        const int dd = 128 * j + q4 * 32 + (lane & ~1);  // even dim of this lane's pair
        const bool rot = a.rotate_out && dd >= rope_lo;
        float c = 1.f, sn = 0.f;
        if (rot) {
          c = d->cs[(dd - rope_lo) >> 1];
          sn = d->sn[(dd - rope_lo) >> 1];
        }
#pragma unroll
        for (int i = 0; i < kHalf / 2; ++i) {
          const float keep = odd ? o[i + kHalf / 2] : o[i];
          const float recv = __shfl_xor_sync(0xffffffffu, odd ? o[i] : o[i + kHalf / 2], 1);
          float x0 = (odd ? recv : keep) * il[i];  // dim dd
          float x1 = (odd ? keep : recv) * il[i];  // dim dd + 1
          if (rot) {
            const float r0 = x0 * c + x1 * sn;
            x1 = x1 * c - x0 * sn;
            x0 = r0;
          }
          *reinterpret_cast<__nv_bfloat162*>(og + (int64_t)(hl + i) * a.dv + dd) = __floats2bfloat162_rn(x0, x1);
        }
      }
      tc::tc_fence_before();
      tc::named_bar_sync(bar_id, 128);
      if (st == 0) tc::mbar_arrive(&ms->dfree[slot]);
    }
    if (!ok && st == 0) atomicExch(&g_attn_tc_error, 5);
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Rows of D bf16 values; boxes of 64 columns x box_rows rows with the 128-byte swizzle.
bool make_row_map(CUtensorMap* m, const void* base, int D, int64_t rows, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows < 1) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

}  // namespace

// Merge the key splits of one (query, head): o = sum_s 2^{m_s - M} O_s / (2^{sink - M} +
// sum_s 2^{m_s - M} l_s), then the -qpos rotation of the rope slice.  One CTA of dv/4
// threads per (query, kCombineHeads heads); thread = 4 consecutive channels of each head, so
// that a thread has the loads of several heads in flight (4 heads per CTA instead of 1: decode
// attention with the combine 88.7 -> 85.2 us).
constexpr int kCombineHeads = 4;

__global__ void __launch_bounds__(128) attn_split_combine_kernel(const AttnArgs a, const TcParams P) {
  const int64_t qrow = blockIdx.x / (kH / kCombineHeads);
  const int hb = (int)(blockIdx.x % (kH / kCombineHeads)) * kCombineHeads;
  const int t4 = threadIdx.x;  // channels 4*t4 .. 4*t4+3
  if (4 * t4 >= a.dv) return;
  const int64_t stride = (int64_t)kH * (a.dv + 2);
  const float* base = a.part + qrow * a.nsplit * stride;
  const int rope_lo = a.D - a.R;
  const bool rot = a.rotate_out && 4 * t4 >= rope_lo;
  float cs[2] = {1.f, 1.f}, sn[2] = {0.f, 0.f};
  if (rot) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int kp = (4 * t4 + 2 * e - rope_lo) >> 1;
      double ang = (double)a.qpos[qrow] * P.inv_freq[kp];
      ang -= rint(ang * 0.15915494309189535) * 6.283185307179586;
      sincosf((float)ang, &sn[e], &cs[e]);
    }
  }
  float M[kCombineHeads], L[kCombineHeads];
  float4 acc[kCombineHeads];
#pragma unroll
  for (int k = 0; k < kCombineHeads; ++k) {
    M[k] = a.sink[hb + k] * kLog2e;
    acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int sp = 0; sp < a.nsplit; ++sp)
#pragma unroll
    for (int k = 0; k < kCombineHeads; ++k) M[k] = fmaxf(M[k], base[sp * stride + (int64_t)kH * a.dv + 2 * (hb + k)]);
#pragma unroll
  for (int k = 0; k < kCombineHeads; ++k) L[k] = tc::ex2(a.sink[hb + k] * kLog2e - M[k]);
  for (int sp = 0; sp < a.nsplit; ++sp) {
#pragma unroll
    for (int k = 0; k < kCombineHeads; ++k) {
      const float* ml = base + sp * stride + (int64_t)kH * a.dv + 2 * (hb + k);
      const float w = tc::ex2(ml[0] - M[k]);
      L[k] += w * ml[1];
      const float4 v = *reinterpret_cast<const float4*>(base + sp * stride + (int64_t)(hb + k) * a.dv + 4 * t4);
      acc[k].x += w * v.x;
      acc[k].y += w * v.y;
      acc[k].z += w * v.z;
      acc[k].w += w * v.w;
    }
  }
#pragma unroll
  for (int k = 0; k < kCombineHeads; ++k) {
    const float inv = 1.f / L[k];
    float x[4] = {acc[k].x * inv, acc[k].y * inv, acc[k].z * inv, acc[k].w * inv};
    if (rot) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float x0 = x[2 * e], x1 = x[2 * e + 1];
        x[2 * e] = x0 * cs[e] + x1 * sn[e];
        x[2 * e + 1] = x1 * cs[e] - x0 * sn[e];
      }
    }
    __nv_bfloat162 b0 = __floats2bfloat162_rn(x[0], x[1]), b1 = __floats2bfloat162_rn(x[2], x[3]);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&b0);
    pk.y = *reinterpret_cast<uint32_t*>(&b1);
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.out) + (qrow * kH + hb + k) * a.dv + 4 * t4) = pk;
  }
}

cudaError_t take_attn_tc_error(int* code) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_attn_tc_error, sizeof(int));
  if (e != cudaSuccess) return e;
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_attn_tc_error, &zero, sizeof(int));
  }
  *code = v;
  return e;
}

bool attn_tc_selects(const AttnArgs& a, int dtype) {
  return a.P_cap >= 1 && a.P_cap <= kSelKeys && a.topk >= 1 && a.topk <= kSelK && a.pool &&
         attn_tc_supported(a, dtype);
}

bool attn_tc_supported(const AttnArgs& a, int dtype) {
  if (dtype != DSV4_BF16 || a.H != kH) return false;
  if (a.D % 64 != 0 || a.D < 128 || a.D > 576) return false;
  if (a.dv % 128 != 0 || a.dv > 512 || a.dv > a.D) return false;
  if (a.D > 512 && a.dv > a.D - 64) return false;  // P^T aliases the last K chunk
  if (a.R > 128 || (a.R & 1) || ((a.D - a.R) % 8) != 0) return false;
  if (!a.pool && a.P_cap > 0) return false;
  return encode_fn() != nullptr;
}

cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t st) {
  const int64_t rows = (int64_t)a.B * a.Sq;
  if (rows == 0) return cudaSuccess;
  CUtensorMap mq;
  if (!make_row_map(&mq, a.q, a.D, rows * kH, kH)) return cudaErrorInvalidValue;
  TcParams P;
  P.a = a;
  if (!P.a.part) P.a.nsplit = 1;
  P.nrows = rows;
  P.nitems = rows * P.a.nsplit;
  for (int k = 0; k < 64; ++k) P.inv_freq[k] = (a.R > 0 && k < a.R / 2) ? pow((double)a.theta, -2.0 * k / a.R) : 0.0;
  // maps for tiles of consecutive rows: the window rows when they are not a ring, the pool
  // when there are no index lists (row coordinates stay below 2^31)
  CUtensorMap mwin = mq, mpool = mq;
  const int64_t win_rows = (int64_t)a.B * a.kv_rows, pool_rows = (int64_t)a.B * a.P_cap;
  P.tma_win = a.kv_win && a.n_win > 0 && !a.win_ring && win_rows + kTile < (1ll << 31) &&
              make_row_map(&mwin, a.kv_win, a.D, win_rows, kTile);
  P.tma_pool = a.pool && !a.idx && !a.scores && a.P_cap > 0 && pool_rows + kTile < (1ll << 31) &&
               make_row_map(&mpool, a.pool, a.D, pool_rows, kTile);
  const Smem L = smem_layout(a.D);
  auto* kern = a.scores ? attn_tc_kernel<true> : attn_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (e != cudaSuccess) return e;
  const int nsm = num_sms();
  const int64_t grid = P.nitems < nsm ? P.nitems : nsm;
  kern<<<(unsigned)grid, kThreads, L.total, st>>>(mq, mwin, mpool, P);
  note_launch();
  if (P.a.nsplit > 1) {
    attn_split_combine_kernel<<<(unsigned)(rows * (kH / kCombineHeads)), 128, 0, st>>>(P.a, P);
    note_launch();
  }
  return cudaGetLastError();
}

int attn_splits(int64_t rows, int64_t keys_per_query) {
  // Split each query's key tiles over CTAs only when there are fewer queries than SMs.  The
  // split minimises the persistent CTAs' critical path, modelled on B200 measurements: ~6 us
  // per 128-key tile, ~2.5 us per work item (the epilogue writing its fp32 partials) and
  // ~0.04 us of HBM time per partial (written, then read by the combine kernel).
  constexpr int64_t kSms = 148;
  if (rows <= 0 || rows >= kSms) return 1;
  const int64_t tiles = keys_per_query > 0 ? (keys_per_query + kTile - 1) / kTile : 1;
  int best = 1;
  double best_cost = 0.0;
  for (int sp = 1; sp <= 16; ++sp) {
    const int64_t items = rows * sp;
    const int64_t per_cta = (items + kSms - 1) / kSms;
    const int64_t tiles_item = (tiles + sp - 1) / sp;
    const double cost = per_cta * (6.0 * tiles_item + 2.5) + (sp > 1 ? 0.04 * items : 0.0);
    if (sp == 1 || cost < best_cost) {
      best_cost = cost;
      best = sp;
    }
  }
  return best;
}

size_t attn_split_bytes(int64_t rows, int64_t keys_per_query, int dv) {
  const int s = attn_splits(rows, keys_per_query);
  return s > 1 ? (size_t)rows * s * kH * (dv + 2) * sizeof(float) : 0;
}

}  // namespace dsv4
