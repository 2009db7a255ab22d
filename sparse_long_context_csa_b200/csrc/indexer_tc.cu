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
#include <cuda.h>
#include <cstddef>
#include <cstdint>
#include <vector>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
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
};

struct IdxSmem {
  uint32_t a, b, misc, total;
};

__host__ __device__ inline IdxSmem idx_smem_layout(int cI, int Npad) {
  IdxSmem s;
  const int nch = cI / 64;
  s.a = 0;                                          // kStages x nch x 16 KB
  s.b = s.a + kStages * nch * 16384;                // nch x Npad x 128 B
  s.misc = s.b + nch * ((Npad * 128 + 1023) / 1024) * 1024;
  s.total = s.misc + 4096;
  return s;
}

struct IdxMisc {
  uint64_t full[kStages], empty[kStages], tfull[2], tempty[2];
  uint32_t tmem_base;
  int maxvis;
  int abort_flag;
  int vis[256];
  alignas(16) float w[256 + 32];  // (query, head) weights, read as float4; zero past the group
};
static_assert(sizeof(IdxMisc) <= 4096, "misc block exceeds its reservation");
static_assert(offsetof(IdxMisc, w) % 16 == 0, "weights are read as float4");

// Scores of one 32-column chunk of the accumulator (columns c .. c+31, column = q * NI + h)
// for the entry of this thread: whole queries for NI <= 32; for NI = 64 two chunks make one
// query (the first leaves its partial sum in `carry`).
template <int NI>
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
#pragma unroll
    for (int qq = 0; qq < 32 / NI; ++qq) {
      float sc = 0.f;
#pragma unroll
      for (int h = 0; h < NI; ++h) sc = fmaf(wv[qq * NI + h], fmaxf(acc[qq * NI + h], 0.f), sc);
      const int q = c / NI + qq;
      if (q < nq && w < vis[q]) sbase[(int64_t)q * P_cap] = sc;
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
      if (q < nq && w < vis[q]) sbase[(int64_t)q * P_cap] = carry + s0 + s1;
    }
  }
}

// The epilogue of one tile for this thread's chunks [k_lo, k_hi) of 32 columns.
template <int NI>
__device__ __forceinline__ void score_tile(uint32_t taddr, int k_lo, int k_hi, const float* wsm, const int* vis,
                                           int nq, int w, float* sbase, int64_t P_cap) {
  float carry = 0.f;
  for (int k = k_lo; k < k_hi; ++k) {
    float acc[32];
    tc::tmem_ld_x32(taddr + 32 * k, acc);
    score_chunk<NI>(acc, 32 * k, wsm, vis, nq, w, sbase, P_cap, carry);
  }
}

__global__ void __launch_bounds__(512, 1) indexer_tc_kernel(const IdxTcParams P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const IndexerArgs& a = P.a;
  const int cI = a.cI, nI = a.nI, QB = P.QB, Npad = P.Npad;
  const int lg_nI = 31 - __clz(nI);
  const int nch = cI / 64;
  const IdxSmem L = idx_smem_layout(cI, Npad);
  IdxMisc* ms = reinterpret_cast<IdxMisc*>(smem + L.misc);
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
            if (w < ms->vis[q]) a.scores[(rbase + q - P.row0) * a.P_cap + w] = sc;
          }
        }
      } else {
        float* sbase = a.scores + (rbase - P.row0) * a.P_cap + w;
        const uint32_t taddr = tmem + tb * Npad + lane_off;
        switch (nI) {
          case 1: score_tile<1>(taddr, k_lo, k_hi, ms->w, ms->vis, nq, w, sbase, a.P_cap); break;
          case 2: score_tile<2>(taddr, k_lo, k_hi, ms->w, ms->vis, nq, w, sbase, a.P_cap); break;
          case 4: score_tile<4>(taddr, k_lo, k_hi, ms->w, ms->vis, nq, w, sbase, a.P_cap); break;
          case 8: score_tile<8>(taddr, k_lo, k_hi, ms->w, ms->vis, nq, w, sbase, a.P_cap); break;
          case 16: score_tile<16>(taddr, k_lo, k_hi, ms->w, ms->vis, nq, w, sbase, a.P_cap); break;
          case 32: score_tile<32>(taddr, k_lo, k_hi, ms->w, ms->vis, nq, w, sbase, a.P_cap); break;
          default: score_tile<64>(taddr, k_lo, k_hi, ms->w, ms->vis, nq, w, sbase, a.P_cap); break;
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
}

}  // namespace

bool indexer_tc_supported(const IndexerArgs& a, int dtype) {
  if (dtype != DSV4_BF16) return false;
  if (a.cI != 64 && a.cI != 128) return false;
  if (a.nI < 1 || a.nI > 64 || (256 % a.nI) != 0) return false;
  return true;
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

cudaError_t launch_indexer_tc_scores(const IndexerArgs& a, int64_t r0, int64_t r1, cudaStream_t st) {
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
  const int nsm = indexer_num_sms();
  int best_tps = max_tiles;
  if (a.q_index) {
    int64_t best_cost = INT64_MAX;
    for (int tps = max_tiles; tps >= 1; --tps) {
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
    for (int tps = max_tiles; tps >= 1; --tps) {
      int64_t n = 0;
      for (int k = 1; k <= max_tiles; ++k) n += groups_with[k] * ((k + tps - 1) / tps);
      const int64_t cost = ((n + nsm - 1) / nsm) * (tps + 2);
      if (cost < best_cost) {
        best_cost = cost;
        best_tps = tps;
      }
    }
  }
  P.tiles_per_split = best_tps;
  const int nsplit = (max_tiles + best_tps - 1) / best_tps;

  const IdxSmem L = idx_smem_layout(a.cI, P.Npad);
  cudaError_t e = cudaFuncSetAttribute(indexer_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)nsplit, (unsigned)ngroups);
  indexer_tc_kernel<<<grid, kThreads, L.total, st>>>(P);
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
