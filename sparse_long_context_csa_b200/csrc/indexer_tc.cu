// Lightning Indexer scores on the sm_100a tensor cores (tcgen05 + TMEM), bf16 inputs.
//
// Method: "DeepSeek-V4" doc, "Hybrid attention (§2.3)" CSA item — the Lightning Indexer
// (eqs. 13-17) scores every query against the compressed indexer-key pool;
// "DeepSeek-V3.2" doc, DSA item 1 — a low-head-count scorer, per-head weights
// (`weights_proj`), computed directly in bf16/fp32 since the Hadamard rotation is
// orthogonal.  Score I[t,w] = sum_h wI[t,h] * relu(qI[t,h] . kI_w).
//
// The query x pool-key product is a dense contraction, so it runs on the tensor cores,
// transposed: D^T[entry, (query, head)] = K_tile[128 x cI] . Qg^T, where Qg holds the
// (query, head) rows of a group of queries (N = queries x heads <= 256).  A TMEM lane is an
// entry, so the ReLU, the head weights and the sum over heads are thread-local in the
// epilogue, and each epilogue thread writes one score per query of the group; rows of 128
// consecutive entries leave coalesced.
//
// Warp roles: 0-3 = producers (entry tiles by 16-byte cp.async into a 4-stage ring; measured
// on B200, TMA boxes of 128-byte rows streamed at ~1.2 TB/s over the whole GPU, cp.async from
// four warps per SM at several times that), 4 = MMA issuer and TMEM owner, 5-12 = epilogue
// (double-buffered TMEM accumulators; two warps per TMEM lane quadrant, each taking half of
// the queries of the group).  The epilogue is specialised on the head count so that every
// 32-column TMEM load turns into whole scores with independent accumulators (measured: a
// generic per-column loop issued ~6x the instructions and held the kernel at 4% of the
// tensor pipe).  Tiles past the largest visible entry count of the group are skipped
// (causality).  Grid: (entry splits, query groups).
//
// Fused top-k (one query per sequence, decode; "DeepSeek-V3.2" doc, DSA item 2: the indices
// go straight to the attention).  The scores of a CTA's split stay in shared memory; after
// scoring, all 16 warps select the split's top-k candidates there (select.cuh), write them
// (order key << 32 | entry) to the work space, and count the split done on a per-query
// counter.  The CTA that counts last merges every split's candidates (keys copied once into
// the free stage buffers) into the query's index row, in ascending entry order.  No CTA waits
// for another, the score rows never reach memory, and the separate top-k launch is gone.  Its
// split of the pool comes from a cost model that also counts the selection and the merge.
#include <cuda.h>
#include <cstddef>
#include <cstdint>
#include <vector>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "select.cuh"
#include "tc_ptx.cuh"

namespace dsv4 {

__device__ int g_indexer_tc_error = 0;

namespace {

constexpr int kThreads = 416;  // 4 producer warps, 1 MMA warp, 8 epilogue warps
constexpr int kEpilogue = 256;
constexpr int kProducers = 128;
constexpr int kStages = 4;
constexpr int kTileE = 128;
constexpr uint32_t kWaitLimit = 1u << 22;

struct IdxTcParams {
  IndexerArgs a;
  int64_t row0, row1;      // rows of this chunk (scores rows are relative to row0)
  int64_t gid0;            // first query group of this launch
  int QB;                  // queries per group
  int Npad;                // QB * nI rounded up to 16
  int tiles_per_split;     // entry tiles per CTA along grid.x
  // fused selection (one query per group): scores stay in shared memory, each CTA keeps its
  // split's top-k candidates (order key << 32 | entry) and the last CTA of a sequence merges
  int select;
  int cand_stride;         // candidates kept per split: min(topk, entries per split)
  uint64_t* cand;          // [rows, gridDim.x, cand_stride] candidates of each split
  int* done;               // [rows] splits finished (zero before the launch; reset by the merge)
};

struct IdxSmem {
  uint32_t a, b, misc, sel, hist, total;
};

// sel_entries: scores kept in shared memory by the fused selection (0: none)
__host__ __device__ inline IdxSmem idx_smem_layout(int cI, int Npad, int sel_entries = 0) {
  IdxSmem s;
  const int nch = cI / 64;
  s.a = 0;                                          // kStages x nch x 16 KB
  s.b = s.a + kStages * nch * 16384;                // nch x Npad x 128 B
  s.misc = s.b + nch * ((Npad * 128 + 1023) / 1024) * 1024;
  s.sel = s.misc + 4096;                            // sel_entries fp32 scores
  s.hist = s.sel + (uint32_t)sel_entries * 4;       // their top-digit histogram (kSelBins words)
  s.total = s.hist + (sel_entries > 0 ? kSelBins * 4 : 0);
  return s;
}

struct IdxMisc {
  uint64_t full[kStages], empty[kStages], tfull[2], tempty[2];
  uint32_t tmem_base;
  int maxvis;
  int minvis;  // the least visible-entry count of the group's rows (0 when a row is past the chunk)
  int abort_flag;
  int sel_last;  // fused selection: this CTA merges the splits of its query
  int vis[256];
  alignas(16) float w[256 + 32];  // (query, head) weights, read as float4; zero past the group
};
static_assert(sizeof(IdxMisc) <= 4096, "misc block exceeds its reservation");
static_assert(offsetof(IdxMisc, w) % 16 == 0, "weights are read as float4");

// Scores of one 32-column chunk of the accumulator (columns c .. c+31, column = q * NI + h)
// for the entry of this thread: whole queries for NI <= 32; for NI = 64 two chunks make one
// query (the first leaves its partial sum in `carry`).  kFull: the tile's entries are visible
// to every query of the group, so no score is masked.
template <int NI, bool kFull>
__device__ __forceinline__ void score_chunk(const float (&acc)[32], int c, const float* wsm, const int* vis, int nq,
                                            int w, float* sbase, int64_t P_cap, float& carry) {
  float wv[32];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float4 v = *reinterpret_cast<const float4*>(wsm + c + 4 * k);
    wv[4 * k] = v.x;
    wv[4 * k + 1] = v.y;
    wv[4 * k + 2] = v.z;
    wv[4 * k + 3] = v.w;
  }
  if constexpr (NI <= 32) {
    float* out = sbase + (int64_t)(c / NI) * P_cap;
#pragma unroll
    for (int qq = 0; qq < 32 / NI; ++qq) {
      float sc = 0.f;
#pragma unroll
      for (int h = 0; h < NI; ++h) sc = fmaf(wv[qq * NI + h], fmaxf(acc[qq * NI + h], 0.f), sc);
      const int q = c / NI + qq;
      if (kFull || (q < nq && w < vis[q])) *out = sc;
      out += P_cap;
    }
  } else {
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int h = 0; h < 32; h += 2) {
      s0 = fmaf(wv[h], fmaxf(acc[h], 0.f), s0);
      s1 = fmaf(wv[h + 1], fmaxf(acc[h + 1], 0.f), s1);
    }
    if ((c & 63) == 0) {
      carry = s0 + s1;
    } else {
      const int q = c / 64;
      if (kFull || (q < nq && w < vis[q])) sbase[(int64_t)q * P_cap] = carry + s0 + s1;
    }
  }
}

// The epilogue of one tile for this thread's chunks [k_lo, k_hi) of 32 columns.
template <int NI>
__device__ __forceinline__ void score_tile(uint32_t taddr, int k_lo, int k_hi, const float* wsm, const int* vis,
                                           int nq, int w, float* sbase, int64_t P_cap, bool full) {
  float carry = 0.f;
  for (int k = k_lo; k < k_hi; ++k) {
    float acc[32];
    tc::tmem_ld_x32(taddr + 32 * k, acc);
    if (full)
      score_chunk<NI, true>(acc, 32 * k, wsm, vis, nq, w, sbase, P_cap, carry);
    else
      score_chunk<NI, false>(acc, 32 * k, wsm, vis, nq, w, sbase, P_cap, carry);
  }
}

constexpr int kSelThreads = 512;           // threads of the fused selection (all 16 warps)
constexpr int kSelMaxEntries = 16384;      // scores per CTA kept for it (64 KB)
constexpr int kSelKeysOffset = 20480;      // merge: candidate keys after the histogram and shared words
constexpr int64_t kSelMinEntries = int64_t(1) << 20;  // scored entries per launch below which it is not used

__device__ __forceinline__ void sel_sync() { asm volatile("bar.sync 3, 512;" ::: "memory"); }

// The split's top-K candidates (n > K scores in shared memory) from the histogram of their
// top 12-bit digits, built by the epilogue while it scored: the digit holding the K-th key,
// then one pass in which each warp lists, in entry order, the entries of its segment at or
// above that digit (bit 31 marks those in it), then the remaining 12 and 8 bits, the counts
// and the ordered write over the lists.  Writes the same candidates, in the same order, as
// select_topk.  Returns false, having written nothing, when a list outgrows its `cap`
// entries (the caller then runs select_topk).  Every thread of the selection calls it.
__device__ __forceinline__ bool split_select_listed(const float* ssc, int n, int K, int w0, const uint32_t* shist,
                                                    uint32_t* hist, SelShared<kSelThreads>* sh, uint32_t* lists,
                                                    int cap, uint64_t* cand) {
  constexpr int kWarps = kSelThreads / 32;
  constexpr uint32_t kIn = 0x80000000u;  // list flag: the key is in the threshold digit
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned below = (1u << lane) - 1u;
  int* over = reinterpret_cast<int*>(hist + kSelBins - 1);  // a histogram word, free here
  select_digit<kSelThreads>(shist, K, tid, sh, sel_sync);
  const uint32_t b1 = (uint32_t)sh->bin;
  int need = sh->rest, cnt = sh->cnt;
  if (tid == 0) *over = 0;
  sel_sync();
  uint32_t* lst = lists + warp * cap;
  const int seg = (n + kWarps - 1) / kWarps;
  const int lo = min(n, warp * seg), hi = min(n, lo + seg);
  int len = 0;
  for (int base = lo; base < hi; base += 32) {
    const int i = base + lane;
    const uint32_t dg = i < hi ? order_key(ssc[i]) >> 20 : 0u;
    const bool sel = i < hi && dg >= b1;
    const unsigned bs = __ballot_sync(0xffffffffu, sel);
    const int pos = len + __popc(bs & below);
    if (sel && pos < cap) lst[pos] = (uint32_t)i | (dg == b1 ? kIn : 0u);
    len += __popc(bs);
  }
  if (lane == 0 && len > cap) atomicOr(over, 1);
  sel_sync();
  if (*over) {
    sel_sync();  // every thread has read the flag before select_topk reuses the histogram
    return false;
  }
  uint32_t prefix = b1 << 20, mask = 0xFFF00000u;
  for (int pass = 1; pass < 3 && cnt != need; ++pass) {
    const int shift = pass == 1 ? 8 : 0;
    const uint32_t dmask = pass == 1 ? 0xFFFu : 0xFFu;
    for (int i = tid; i < kSelBins; i += kSelThreads) hist[i] = 0u;
    sel_sync();
    for (int p = lane; p < len; p += 32) {
      const uint32_t e = lst[p];
      if (e & kIn) {
        const uint32_t k = order_key(ssc[e & ~kIn]);
        if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & dmask], 1u);
      }
    }
    sel_sync();
    select_digit<kSelThreads>(hist, need, tid, sh, sel_sync);
    prefix |= (uint32_t)sh->bin << shift;
    mask |= dmask << shift;
    need = sh->rest;
    cnt = sh->cnt;
  }
  // this segment's listed keys above / equal to the final prefix (entries outside the
  // threshold digit are above it), a scan over warps, then the ordered write
  int n_gt = 0, n_eq = 0;
  for (int p = lane; p < len; p += 32) {
    const uint32_t e = lst[p];
    if (e & kIn) {
      const uint32_t k = order_key(ssc[e & ~kIn]) & mask;
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
  if (lane == 0) {
    sh->wcnt_gt[warp] = n_gt;
    sh->wcnt_eq[warp] = n_eq;
  }
  sel_sync();
  int pos_gt = 0, pos_eq = 0;
  for (int w = 0; w < warp; ++w) {
    pos_gt += sh->wcnt_gt[w];
    pos_eq += sh->wcnt_eq[w];
  }
  for (int base = 0; base < len; base += 32) {
    const int p = base + lane;
    const uint32_t e = p < len ? lst[p] : 0u;
    const uint32_t key = p < len ? order_key(ssc[e & ~kIn]) : 0u;
    const bool gt = p < len && (!(e & kIn) || (key & mask) > prefix);
    const bool eq = p < len && (e & kIn) && (key & mask) == prefix;
    const unsigned bgt = __ballot_sync(0xffffffffu, gt), beq = __ballot_sync(0xffffffffu, eq);
    const int my_eq_rank = pos_eq + __popc(beq & below);
    const int slot = pos_gt + __popc(bgt & below) + min(my_eq_rank, need);
    if ((gt || (eq && my_eq_rank < need)) && slot < K)
      cand[slot] = ((uint64_t)key << 32) | (uint32_t)(w0 + (int)(e & ~kIn));
    pos_gt += __popc(bgt);
    pos_eq += __popc(beq);
  }
  sel_sync();
  return true;
}

template <bool kSelect>
__global__ void __launch_bounds__(512, 1) indexer_tc_kernel(const IdxTcParams P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const IndexerArgs& a = P.a;
  const int cI = a.cI, nI = a.nI, QB = P.QB, Npad = P.Npad;
  const int lg_nI = 31 - __clz(nI);
  const int nch = cI / 64;
  const IdxSmem L = idx_smem_layout(cI, Npad, kSelect ? P.tiles_per_split * kTileE : 0);
  IdxMisc* ms = reinterpret_cast<IdxMisc*>(smem + L.misc);
  float* ssc = reinterpret_cast<float*>(smem + L.sel);  // fused selection: this CTA's scores
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((tc::smem_u32(smem) & 1023u) != 0) {
    if (tid == 0) atomicExch(&g_indexer_tc_error, 3);
    return;
  }

  // query group -> sequence and rows
  const int groups_per_seq = (a.Sq + QB - 1) / QB;
  const int64_t gid = P.gid0 + blockIdx.y;
  const int b = (int)(gid / groups_per_seq);
  const int s0 = (int)(gid % groups_per_seq) * QB;
  const int nq = min(QB, a.Sq - s0);
  const int64_t rbase = (int64_t)b * a.Sq + s0;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      tc::mbar_init(&ms->full[i], kProducers);  // one cp.async arrival per producer thread
      tc::mbar_init(&ms->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&ms->tfull[i], 1);
      tc::mbar_init(&ms->tempty[i], kEpilogue);
    }
    ms->maxvis = 0;
    ms->minvis = 0x7fffffff;
    ms->abort_flag = 0;
    tc::mbar_fence_init();
  }
  __syncthreads();
  // per-query visibility and head weights
  for (int q = tid; q < QB; q += kThreads) {
    int v = 0;
    const int64_t row = rbase + q;
    if (q < nq && row >= P.row0 && row < P.row1) {
      const int t = query_cache_index(a.q_index, row, s0 + q);
      v = visible_entries(t, a.m, a.P_cap);
      if (v < 0) v = 0;
    }
    ms->vis[q] = v;
    atomicMax(&ms->maxvis, v);
    atomicMin(&ms->minvis, v);
  }
  for (int i = tid; i < 256 + 32; i += kThreads) ms->w[i] = (i < QB * nI && (i / nI) < nq) ? a.wI[rbase * nI + i] : 0.f;
  __syncthreads();
  // this CTA's entry tiles; a CTA past the group's visible entries leaves before loading
  // anything (finer entry splits of causal prefill groups leave many such CTAs)
  const int maxvis = ms->maxvis;
  const int ntile_all = (maxvis + kTileE - 1) / kTileE;
  const int t_lo = blockIdx.x * P.tiles_per_split;
  const int t_hi = min(ntile_all, t_lo + P.tiles_per_split);
  const int ntiles = t_hi > t_lo ? t_hi - t_lo : 0;
  if (kSelect && ntile_all == 0 && blockIdx.x == 0) {
    // nothing visible yet: the whole row is -1
    int32_t* out = a.idx + rbase * (int64_t)a.topk;
    for (int i = tid; i < a.topk; i += kThreads) out[i] = -1;
  }
  if (ntiles == 0) return;
  if (warp == 4) {
    tc::tmem_alloc(&ms->tmem_base, 2 * Npad <= 32 ? 32 : (2 * Npad <= 64 ? 64 : (2 * Npad <= 128 ? 128 : (2 * Npad <= 256 ? 256 : 512))));
    tc::tmem_relinquish();
  }
  // (query, head) rows -> K-major 128B-swizzled B operand, by cp.async (rows past the group
  // are zero-filled with plain stores)
  {
    const __nv_bfloat16* qI = static_cast<const __nv_bfloat16*>(a.qI);
    const int per_row = cI / 8;  // 16-byte pieces per row
    const uint32_t chunk_bytes = ((Npad * 128 + 1023) / 1024) * 1024;
    for (int ci = tid; ci < Npad * per_row; ci += kThreads) {
      const int r = ci / per_row;
      const int d0 = (ci % per_row) * 8;
      const int ch = d0 / 64, u = (d0 % 64) / 8;
      uint8_t* dst = smem + L.b + ch * chunk_bytes + r * 128 + ((u ^ (r & 7)) * 16);
      if (r < nq * nI)
        tc::cp_async_16(dst, qI + (rbase * nI + r) * cI + d0);
      else
        *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  }
  uint32_t* shist = reinterpret_cast<uint32_t*>(smem + L.hist);  // fused selection: top digits of ssc
  if constexpr (kSelect)
    for (int i = tid; i < kSelBins; i += blockDim.x) shist[i] = 0u;
  tc::fence_proxy_async_smem();
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();

  const uint32_t tmem = ms->tmem_base;
  const uint32_t b_chunk = ((Npad * 128 + 1023) / 1024) * 1024;

  if (warp < 4) {
    // ---------------------------------------------------------------- producers (4 warps)
    // 16-byte cp.async copies of the entry tile straight into the 128B-swizzled layout:
    // per 64-channel chunk, thread t copies unit (t & 7) of rows (t >> 3) + 16j, j < 8.
    const int u = tid & 7;
    const int64_t row_end = (int64_t)a.B * a.P_cap;  // rows past the tensor are not read
    const __nv_bfloat16* poolI = static_cast<const __nv_bfloat16*>(a.poolI);
    for (int i = 0; i < ntiles; ++i) {
      const int st = i % kStages;
      const uint32_t ph = (i / kStages) & 1;
      if (i >= kStages && !tc::mbar_wait(&ms->empty[st], ph ^ 1, kWaitLimit)) {
        atomicExch(&g_indexer_tc_error, 1);
        ms->abort_flag = 1;
      }
      const int64_t r0 = (int64_t)b * a.P_cap + (int64_t)(t_lo + i) * kTileE;
      for (int c = 0; c < nch; ++c) {
        uint8_t* cb = smem + L.a + (st * nch + c) * 16384;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int r = (tid >> 3) + 16 * j;
          if (r0 + r < row_end)
            tc::cp_async_16(cb + r * 128 + ((u ^ (r & 7)) * 16), poolI + (r0 + r) * cI + c * 64 + u * 8);
        }
      }
      tc::cp_async_arrive_noinc(&ms->full[st]);
    }
  } else if (warp == 4) {
    // ---------------------------------------------------------------- MMA issuer
    const uint32_t idesc = tc::idesc_bf16_f32(128, Npad, 0, 0);
    const uint32_t abase = tc::smem_u32(smem + L.a);
    const uint32_t bbase = tc::smem_u32(smem + L.b);
    for (int i = 0; i < ntiles; ++i) {
      const int st = i % kStages;
      const int tb = i & 1;
      if (!__all_sync(0xffffffffu, tc::mbar_wait(&ms->full[st], (i / kStages) & 1, kWaitLimit) &&
                                      ms->abort_flag == 0)) {
        if (lane == 0) atomicExch(&g_indexer_tc_error, 2);
        break;
      }
      tc::fence_proxy_async_smem();  // cp.async wrote the tile through the generic proxy
      if (i >= 2 && !__all_sync(0xffffffffu, tc::mbar_wait(&ms->tempty[tb], ((i >> 1) & 1) ^ 1, kWaitLimit))) {
        if (lane == 0) atomicExch(&g_indexer_tc_error, 4);
        break;
      }
      tc::tc_fence_after();
      if (lane == 0) {
        for (int kk = 0; kk < cI / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint64_t ad = tc::sdesc_sw128(abase + st * nch * 16384 + off, 16, 1024);
          const uint64_t bd = tc::sdesc_sw128(bbase + (kk >> 2) * b_chunk + (kk & 3) * 32, 16, 1024);
          tc::umma_f16(tmem + tb * Npad, ad, bd, idesc, kk > 0 ? 1u : 0u);
        }
        tc::umma_commit(&ms->empty[st]);
        tc::umma_commit(&ms->tfull[tb]);
      }
      __syncwarp();
    }
  } else if (warp >= 13) {
    // fused selection launches: three more warps that only join the selection
  } else {
    // ---------------------------------------------------------------- epilogue (8 warps)
    const int q4 = warp & 3;
    const int half = (warp - 5) >> 2;
    const int e = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    // few columns (decode): weights and visibility live in registers for the whole CTA
    const bool small = Npad == 16;
    float wsm[16];
    int qcol[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      qcol[j] = j >> lg_nI;
      wsm[j] = (small && qcol[j] < nq) ? ms->w[j] : 0.f;
    }
    // 32-column chunks of this half: whole queries (two chunks per query when nI = 64)
    const int nchk = (Npad + 31) / 32;
    const int cpq = nI > 32 ? 2 : 1;
    const int units = (nchk + cpq - 1) / cpq;
    const int u_mid = (units + 1) / 2;
    const int k_lo = half == 0 ? 0 : u_mid * cpq;
    const int k_hi = half == 0 ? min(nchk, u_mid * cpq) : nchk;
    for (int i = 0; i < ntiles; ++i) {
      const int tb = i & 1;
      if (!tc::named_bar_and(1, kEpilogue, tc::mbar_wait(&ms->tfull[tb], (i >> 1) & 1, kWaitLimit))) {
        if (tid == 160) atomicExch(&g_indexer_tc_error, 5);
        break;
      }
      tc::tc_fence_after();
      const int w = (t_lo + i) * kTileE + e;
      if (small) {
        if (half == 0) {
          float acc[16];
          tc::tmem_ld_x16(tmem + tb * Npad + lane_off, acc);
          for (int q = 0; q < nq; ++q) {
            float sc = 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j) sc = fmaf(qcol[j] == q ? wsm[j] : 0.f, fmaxf(acc[j], 0.f), sc);
            if (kSelect) {
              ssc[i * kTileE + e] = sc;  // one query per group; entries past vis are never read
              if (w < ms->vis[q]) atomicAdd(&shist[order_key(sc) >> 20], 1u);
            } else if (w < ms->vis[q])
              a.scores[(rbase + q - P.row0) * a.P_cap + w] = sc;
          }
        }
      } else if constexpr (!kSelect) {  // the fused selection has one query of <= 16 heads: small
        float* sbase = a.scores + (rbase - P.row0) * a.P_cap + w;
        const uint32_t taddr = tmem + tb * Npad + lane_off;
        // every entry of the tile visible to every query of the group (all but the causal
        // diagonal of prefill): no per-score mask
        const bool full = (t_lo + i + 1) * kTileE <= ms->minvis;
        switch (nI) {
          case 1: score_tile<1>(taddr, k_lo, k_hi, ms->w, ms->vis, nq, w, sbase, a.P_cap, full); break;
          case 2: score_tile<2>(taddr, k_lo, k_hi, ms->w, ms->vis, nq, w, sbase, a.P_cap, full); break;
          case 4: score_tile<4>(taddr, k_lo, k_hi, ms->w, ms->vis, nq, w, sbase, a.P_cap, full); break;
          case 8: score_tile<8>(taddr, k_lo, k_hi, ms->w, ms->vis, nq, w, sbase, a.P_cap, full); break;
          case 16: score_tile<16>(taddr, k_lo, k_hi, ms->w, ms->vis, nq, w, sbase, a.P_cap, full); break;
          case 32: score_tile<32>(taddr, k_lo, k_hi, ms->w, ms->vis, nq, w, sbase, a.P_cap, full); break;
          default: score_tile<64>(taddr, k_lo, k_hi, ms->w, ms->vis, nq, w, sbase, a.P_cap, full); break;
        }
      }
      tc::tc_fence_before();
      tc::mbar_arrive(&ms->tempty[tb]);
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 2 * Npad <= 32 ? 32 : (2 * Npad <= 64 ? 64 : (2 * Npad <= 128 ? 128 : (2 * Npad <= 256 ? 256 : 512))));
  }
  if constexpr (kSelect) {
    if (tid >= kSelThreads) return;
    // ------------------------------------------------------------ split top-k (warps 0-7)
    // The pipeline's stage buffers are free now: they hold the radix histogram and the
    // selection's shared words.
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem + L.a);
    SelShared<kSelThreads>* sh = reinterpret_cast<SelShared<kSelThreads>*>(smem + L.a + kSelBins * 4);
    const int K = a.topk;
    const int vis = ms->vis[0];
    const int per = P.tiles_per_split * kTileE;  // entries per split
    const int w0 = t_lo * kTileE;
    const int n_loc = min(ntiles * kTileE, vis - w0);
    const int stride = P.cand_stride;
    uint64_t* cand = P.cand + ((int64_t)(rbase - P.row0) * gridDim.x + blockIdx.x) * stride;
    if (n_loc <= K) {
      for (int i = tid; i < n_loc; i += kSelThreads)
        cand[i] = ((uint64_t)order_key(ssc[i]) << 32) | (uint32_t)(w0 + i);
    } else if (!split_select_listed(ssc, n_loc, K, w0, shist, hist, sh,
                                    reinterpret_cast<uint32_t*>(smem + L.a + kSelKeysOffset),
                                    (kStages * nch * 16384 - kSelKeysOffset) / 4 / (kSelThreads / 32), cand)) {
      select_topk<kSelThreads>(
          n_loc, K, tid, [&](int i) { return order_key(ssc[i]); },
          [&](int slot, int i) { cand[slot] = ((uint64_t)order_key(ssc[i]) << 32) | (uint32_t)(w0 + i); }, hist, sh,
          sel_sync);
    }
    // the last split of this query to finish merges (no CTA waits for another)
    __threadfence();
    sel_sync();
    const int nonempty = (ntile_all + P.tiles_per_split - 1) / P.tiles_per_split;
    if (tid == 0) ms->sel_last = atomicAdd(&P.done[rbase - P.row0], 1) == nonempty - 1;
    sel_sync();
    if (!ms->sel_last) return;
    __threadfence();
    // the candidates of all splits in split order (ascending entries): every split but the
    // last holds `stride` of them, the last min(topk, its visible entries); read through L2
    const uint64_t* all = P.cand + (int64_t)(rbase - P.row0) * gridDim.x * stride;
    const int full = (nonempty - 1) * stride;
    const int n_tot = full + min(K, vis - (nonempty - 1) * per);
    auto cand_at = [&](int i) {
      const int sp = i < full ? i / stride : nonempty - 1;
      return __ldcg(all + (int64_t)sp * stride + (i - sp * stride));
    };
    int32_t* out = a.idx + rbase * (int64_t)K;
    if (n_tot <= K) {
      for (int i = tid; i < K; i += kSelThreads) out[i] = i < n_tot ? (int32_t)(uint32_t)cand_at(i) : -1;
    } else {
      // the candidates' keys go to shared memory once (after the histogram and the shared
      // words, in the free stage buffers); the radix passes then read them from there
      uint32_t* mk = reinterpret_cast<uint32_t*>(smem + L.a + kSelKeysOffset);
      for (int sp = 0; sp < nonempty; ++sp) {
        const int nc = sp < nonempty - 1 ? stride : n_tot - full;
        const uint64_t* src = all + (int64_t)sp * stride;
        uint32_t* dst = mk + sp * stride;
        for (int i0 = 0; i0 < nc; i0 += 8 * kSelThreads) {  // eight loads in flight per thread
          uint64_t v[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * kSelThreads + tid;
            v[u] = i < nc ? __ldcg(src + i) : 0ull;
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * kSelThreads + tid;
            if (i < nc) dst[i] = (uint32_t)(v[u] >> 32);
          }
        }
      }
      sel_sync();
      select_topk<kSelThreads>(
          n_tot, K, tid, [&](int i) { return mk[i]; },
          [&](int slot, int i) { out[slot] = (int32_t)(uint32_t)cand_at(i); }, hist, sh, sel_sync);
    }
    if (tid == 0) P.done[rbase - P.row0] = 0;  // ready for the next launch
  }
}

}  // namespace

bool indexer_tc_supported(const IndexerArgs& a, int dtype) {
  if (dtype != DSV4_BF16) return false;
  if (a.cI != 64 && a.cI != 128) return false;
  if (a.nI < 1 || a.nI > 64 || (256 % a.nI) != 0) return false;
  return true;
}

// Shared memory one CTA may opt in to on the current device (cached per device).
int indexer_smem_optin() {
  static int per_dev[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (per_dev[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess || v <= 0) return 0;
    per_dev[dev] = v;
  }
  return per_dev[dev];
}

int indexer_num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

// Launch plan of the tensor-core indexer over rows [r0, r1) on nsm SMs; max_tps caps the entry
// tiles per CTA (0: no cap).
static IdxTcParams plan_indexer_tc(const IndexerArgs& a, int64_t r0, int64_t r1, int max_tps, int nsm,
                                   dim3* grid_out, bool select = false) {
  IdxTcParams P{};
  P.a = a;
  P.row0 = r0;
  P.row1 = r1;
  // queries per group: fill N = 256 when the sequence is long enough; decode groups are one query
  int QB = 256 / a.nI;
  if (QB > a.Sq) QB = a.Sq;
  P.QB = QB;
  P.Npad = ((QB * a.nI + 15) / 16) * 16;
  const int gps = (a.Sq + QB - 1) / QB;
  const int64_t g_lo = (r0 / a.Sq) * gps + (r0 % a.Sq) / QB;
  const int64_t g_hi = ((r1 - 1) / a.Sq) * gps + ((r1 - 1) % a.Sq) / QB + 1;
  P.gid0 = g_lo;
  const int64_t ngroups = g_hi - g_lo;
  const int max_tiles = (a.P_cap + kTileE - 1) / kTileE;
  // Split the entry axis when there are too few query groups to fill the GPU.  One CTA fits
  // per SM, so CTAs run in waves of the SM count.  With cache indices (decode) every group
  // scans about the whole pool: pick the tiles per CTA that minimise waves x (tiles per CTA
  // + a set-up cost of about two tiles), so that the last wave is not left mostly empty
  // (measured: 320 CTAs in 2.2 waves held the decode indexer to 63% of HBM bandwidth).
  // Prefill (no cache indices) is causal: tile counts grow along the groups and are known
  // here, so the same cost is evaluated over the CTAs that have work.
  int best_tps = max_tiles;
  const int tps_hi = max_tps > 0 && max_tps < max_tiles ? max_tps : max_tiles;
  if (a.q_index && select) {
    // fused selection, in units of one scored tile (measured on B200, decode shapes): a split
    // selects over its entries at ~1/4 tile per tile it scored, and the last split of a query
    // merges every split's min(topk, entries) candidates at ~1/400 tile per candidate
    double best_cost = 1e300;
    for (int tps = tps_hi; tps >= 1; --tps) {
      const int ns = (max_tiles + tps - 1) / tps;
      const int64_t waves = (ngroups * ns + nsm - 1) / nsm;
      const int stride = a.topk < tps * kTileE ? a.topk : tps * kTileE;
      const double cost = waves * (1.25 * tps + 2.0) + (ns > 1 ? 0.0026 * ns * stride : 0.0);
      if (cost < best_cost) {
        best_cost = cost;
        best_tps = tps;
      }
    }
  } else if (a.q_index) {
    int64_t best_cost = INT64_MAX;
    for (int tps = tps_hi; tps >= 1; --tps) {
      const int ns = (max_tiles + tps - 1) / tps;
      const int64_t waves = (ngroups * ns + nsm - 1) / nsm;
      const int64_t cost = waves * (tps + 2);
      if (cost < best_cost) {
        best_cost = cost;
        best_tps = tps;
      }
    }
  } else {
    // causal prefill: group g needs ceil(min((s0 + nq) / m, P_cap) / 128) tiles; CTAs past
    // them exit at once, so the cost counts the non-empty CTAs only
    std::vector<int64_t> groups_with(max_tiles + 1, 0);  // number of groups needing k tiles
    for (int64_t g = g_lo; g < g_hi; ++g) {
      const int gs0 = (int)(g % gps) * QB;
      const int gnq = QB < a.Sq - gs0 ? QB : a.Sq - gs0;
      int mv = (gs0 + gnq) / a.m;
      if (mv > a.P_cap) mv = a.P_cap;
      ++groups_with[(mv + kTileE - 1) / kTileE];
    }
    int64_t best_cost = INT64_MAX;
    for (int tps = tps_hi; tps >= 1; --tps) {
      int64_t n = 0;
      for (int k = 1; k <= max_tiles; ++k) n += groups_with[k] * ((k + tps - 1) / tps);
      const int64_t cost = ((n + nsm - 1) / nsm) * (tps + 2);
      if (cost < best_cost) {
        best_cost = cost;
        best_tps = tps;
      }
    }
  }
  if (max_tps > 0 && best_tps > max_tps) best_tps = max_tps;
  P.tiles_per_split = best_tps;
  const int nsplit = (max_tiles + best_tps - 1) / best_tps;
  *grid_out = dim3((unsigned)nsplit, (unsigned)ngroups);
  return P;
}

cudaError_t launch_indexer_tc_scores(const IndexerArgs& a, int64_t r0, int64_t r1, cudaStream_t st) {
  dim3 grid;
  const IdxTcParams P = plan_indexer_tc(a, r0, r1, 0, indexer_num_sms(), &grid);
  const IdxSmem L = idx_smem_layout(a.cI, P.Npad);
  cudaError_t e =
      cudaFuncSetAttribute(indexer_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (e != cudaSuccess) return e;
  indexer_tc_kernel<false><<<grid, kThreads, L.total, st>>>(P);
  note_launch();
  return cudaGetLastError();
}

// Fused scores + top-k for one query per sequence (decode): split top-k in each CTA, merged by
// the last CTA of each query.  Work space (a.scores, ws_bytes): the per-query split counters,
// then the candidates.  Returns cudaErrorNotSupported when the shapes or the work space do
// not allow it (the caller then runs the two kernels).
// (planned for the 148 SMs of a B200, so that the size is a function of the sizes alone; on
// another SM count the plan may need more and the two-kernel path runs instead)
size_t indexer_tc_select_bytes(const IndexerArgs& a, int64_t rows) {
  if (a.Sq != 1 || a.nI > 16 || rows < 1) return 0;
  dim3 grid;
  const IdxTcParams P = plan_indexer_tc(a, 0, rows, kSelMaxEntries / kTileE, 148, &grid, true);
  const int per = P.tiles_per_split * kTileE;
  const size_t stride = (size_t)(a.topk < per ? a.topk : per);
  return ((size_t)rows * sizeof(int) + 255) / 256 * 256 + (size_t)rows * grid.x * stride * sizeof(uint64_t);
}

cudaError_t launch_indexer_tc_select(const IndexerArgs& a, int64_t r0, int64_t r1, size_t ws_bytes,
                                     cudaStream_t st) {
  if (a.Sq != 1 || a.nI > 16 || !a.idx) return cudaErrorNotSupported;
  // Measured on B200: the fused kernel is ahead from about a million scored entries per launch
  // (64 queries x 32768 entries: 144 us against 152 us for the two kernels), behind below it
  // (32 x 15000: 67 against 60 us), where too few splits leave SMs idle.
  if ((r1 - r0) * (int64_t)a.P_cap < kSelMinEntries) return cudaErrorNotSupported;
  dim3 grid;
  IdxTcParams P = plan_indexer_tc(a, r0, r1, kSelMaxEntries / kTileE, indexer_num_sms(), &grid, true);
  if (P.QB != 1) return cudaErrorNotSupported;
  const int64_t rows = r1 - r0;
  const int nsplit = (int)grid.x;
  const int per = P.tiles_per_split * kTileE;
  P.cand_stride = a.topk < per ? a.topk : per;
  // the merge keeps every split's candidate keys in the stage buffers
  const int64_t merge_keys = (int64_t)nsplit * P.cand_stride;
  if (merge_keys * 4 > (int64_t)kStages * (a.cI / 64) * 16384 - kSelKeysOffset) return cudaErrorNotSupported;
  const size_t done_bytes = ((size_t)rows * sizeof(int) + 255) / 256 * 256;
  const size_t need = done_bytes + (size_t)rows * nsplit * P.cand_stride * sizeof(uint64_t);
  if (need > ws_bytes) return cudaErrorNotSupported;
  P.select = 1;
  P.done = reinterpret_cast<int*>(a.scores);
  P.cand = reinterpret_cast<uint64_t*>(reinterpret_cast<char*>(a.scores) + done_bytes);
  const IdxSmem L = idx_smem_layout(a.cI, P.Npad, P.tiles_per_split * kTileE);
  // the kept scores and their histogram take 80 KB more shared memory than the score kernel;
  // a device that cannot give a CTA that much runs the two kernels instead
  if ((int64_t)L.total > indexer_smem_optin()) return cudaErrorNotSupported;
  cudaError_t e = cudaMemsetAsync(P.done, 0, (size_t)rows * sizeof(int), st);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(indexer_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (e != cudaSuccess) return e;
  indexer_tc_kernel<true><<<grid, kSelThreads, L.total, st>>>(P);
  note_launch();
  return cudaGetLastError();
}

cudaError_t take_indexer_tc_error(int* code) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_indexer_tc_error, sizeof(int));
  if (e != cudaSuccess) return e;
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_indexer_tc_error, &zero, sizeof(int));
  }
  *code = v;
  return e;
}

}  // namespace dsv4

