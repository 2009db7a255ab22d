// Sparse shared-K=V MQA attention with sink on the sm_100a tensor cores (tcgen05 + TMEM),
// bf16 inputs, fp32 accumulation.
//
// Method: "DeepSeek-V4" doc, "Hybrid attention (§2.3)" — one K=V head read as both key and
// value, partial interleaved RoPE with the -i rotation of the output rope slice (eq. 26),
// per-head sink (eq. 27), the sliding-window K=V rows concatenated with the compressor
// entries picked by the Lightning Indexer; "DeepSeek-V3.2" doc, DSA item 2 (attention over
// the selected tokens only).
//
// Design (one CTA per query token; its 64 heads share every key row):
//  * The key set of a query (window rows, then the selected pool entries) is cut into
//    tiles of 128 keys.  One producer warp gathers a tile's rows with TMA tile::gather4
//    (4 arbitrary rows per instruction, 128-byte swizzle) straight into the operand layout.
//  * Scores are computed transposed, S^T[key, head] = K_tile . Q^T, as one 128x64xD MMA
//    chain (M = 128 keys keeps the tensor core at full rate; 64 heads alone would be an
//    M=64 half-rate shape).  The same shared-memory tile is then read as V^T (MN-major)
//    for O^T[dim, head] += V^T . P^T: K=V costs one gather for both products.
//  * The softmax warps own one key (TMEM lane) each and hold its 64 head scores.  The
//    running max per head starts at the sink logit and is only raised when some score
//    exceeds it by more than 2^8 (then the O^T columns are rescaled in TMEM), so the common
//    tile needs no cross-thread reduction.  Per-thread partial denominators are reduced
//    once, in the epilogue, where the sink term e^{sink - max} is added.
//  * Accumulators: S^T 64 TMEM columns, O^T dv/128 tiles x 64 columns.
//  * The output leaves TMEM transposed; it is staged through shared memory and written
//    with 16-byte coalesced stores, after the -qpos rotation of the rope slice.
// Warp roles: 0 = TMA producer, 1 = MMA issuer (and TMEM owner), 2-5 = softmax/epilogue.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "tc_ptx.cuh"

namespace dsv4 {

__device__ int g_attn_tc_error = 0;  // non-zero: a pipeline wait gave up (the CTA returned early)

namespace {

constexpr int kH = 64;
constexpr int kTile = 128;
constexpr int kThreads = 192;
constexpr int kSoftmaxWarp0 = 2;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: p <= 2^8 between rescales
constexpr uint32_t kWaitLimit = 1u << 22;

struct Smem {
  // byte offsets inside the dynamic shared memory window
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
  s.total = s.misc + 4096;
  return s;
}

struct Misc {
  uint64_t kfull, sfull, pfull, odone;
  uint32_t tmem_base;
  int npool_last;   // highest valid pool slot + 1
  int abort_flag;
  int rescale_cnt[2];
  uint32_t mask[4];     // validity of the 128 keys of the current tile
  float m[kH];          // running max per head (log2 units)
  float cs[64], sn[64]; // RoPE table of the query position
  float inv_l[kH];
  float fac[kH];        // rescale factor per head (rare path)
  float red[4][kH];
};
static_assert(sizeof(Misc) <= 4096, "misc block exceeds its reservation");

__device__ __forceinline__ void set_error(Misc* ms, int code) {
  atomicExch(&g_attn_tc_error, code);
  ms->abort_flag = 1;
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap map_win, const __grid_constant__ CUtensorMap map_pool,
                   const AttnArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int D = a.D;
  const int nch = D / 64;
  const Smem L = smem_layout(D);
  Misc* ms = reinterpret_cast<Misc*>(smem + L.misc);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if ((tc::smem_u32(smem) & 1023u) != 0) {  // the swizzle atoms need a 1024-byte aligned base
    if (tid == 0) atomicExch(&g_attn_tc_error, 3);
    return;
  }

  const int64_t qrow = blockIdx.x;
  const int b = (int)(qrow / a.Sq);
  const int s = (int)(qrow % a.Sq);
  const int t = query_cache_index(a.q_index, qrow, s);
  const int vis = visible_entries(t, a.m, a.P_cap);
  const int wlo = t - a.n_win + 1 > 0 ? t - a.n_win + 1 : 0;
  const int win_rows = a.win_ring ? a.win_ring : a.kv_rows;
  int nw = a.n_win > 0 ? t - wlo + 1 : 0;
  if (nw < 0) nw = 0;
  if (!a.win_ring && wlo + nw > a.kv_rows) nw = a.kv_rows > wlo ? a.kv_rows - wlo : 0;
  const int nw4 = (nw + 3) & ~3;

  // ---------------------------------------------------------------- prologue
  if (tid == 0) {
    tc::mbar_init(&ms->kfull, 1);
    tc::mbar_init(&ms->sfull, 1);
    tc::mbar_init(&ms->pfull, 128);
    tc::mbar_init(&ms->odone, 1);
    ms->npool_last = a.idx ? 0 : (vis > 0 ? vis : 0);
    ms->abort_flag = 0;
    ms->rescale_cnt[0] = ms->rescale_cnt[1] = 0;
    tc::mbar_fence_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&ms->tmem_base, 512);
    tc::tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tensormap(&map_win);
    tc::prefetch_tensormap(&map_pool);
  }
  // RoPE table of the query position
  const int R = a.R;
  if (a.rope_q || a.rotate_out) {
    for (int k = tid; k < R / 2; k += kThreads) {
      float c, sn;
      rope_cos_sin(a.qpos[qrow], k, R, a.theta, &c, &sn);
      ms->cs[k] = c;
      ms->sn[k] = sn;
    }
  }
  for (int h = tid; h < kH; h += kThreads) ms->m[h] = a.sink[h] * kLog2e;
  __syncthreads();
  // last valid pool slot (slots past it are not processed; holes inside are masked)
  if (a.idx) {
    int last = 0;
    const int32_t* ir = a.idx + qrow * a.topk;
    for (int k = tid; k < a.topk; k += kThreads) {
      const int w = ir[k];
      if (w >= 0 && w < vis) last = k + 1;
    }
    if (last) atomicMax(&ms->npool_last, last);
  }
  // q rows (64 heads x D), rotated at qpos, into the 128B-swizzled K-major B-operand layout
  {
    const uint4* qg = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.q) + qrow * kH * D);
    const int per_head = D / 8;
    const int rope_lo = D - R;
    for (int ci = tid; ci < kH * per_head; ci += kThreads) {
      const int h = ci / per_head;
      const int d0 = (ci % per_head) * 8;
      uint4 v = qg[ci];
      if (a.rope_q && d0 >= rope_lo) {
        __nv_bfloat162* p2 = reinterpret_cast<__nv_bfloat162*>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(p2[e]);
          const int k = (d0 - rope_lo) / 2 + e;
          const float c = ms->cs[k], sn = ms->sn[k];
          p2[e] = __floats2bfloat162_rn(f.x * c - f.y * sn, f.x * sn + f.y * c);
        }
      }
      const int ch = d0 / 64, u = (d0 % 64) / 8;
      *reinterpret_cast<uint4*>(smem + L.q + ch * 8192 + h * 128 + ((u ^ (h & 7)) * 16)) = v;
    }
  }
  tc::fence_proxy_async_smem();
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();

  const int npool = ms->npool_last;
  const int NK = nw4 + npool;
  const int ntiles = (NK + kTile - 1) / kTile;
  const uint32_t tmem = ms->tmem_base;
  const uint32_t tS = tmem, tO = tmem + 64;
  const int nvt = a.dv / 128;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    const int32_t* ir = a.idx ? a.idx + qrow * a.topk : nullptr;
    const int win_base = b * win_rows;
    const int pool_base = b * a.P_cap;
    for (int i = 0; i < ntiles; ++i) {
      // every lane takes the same decision, so no lane is left waiting in __syncwarp
      if (!__all_sync(0xffffffffu, i == 0 || tc::mbar_wait(&ms->odone, (i - 1) & 1, kWaitLimit))) {
        if (lane == 0) set_error(ms, 1);
        break;
      }
      const int k0 = i * kTile;
      const int nvalid = min(kTile, NK - k0);
      const int nk = (nvalid + 15) & ~15;
      // validity mask of the tile (lane l covers keys 4l..4l+3)
      uint32_t bits = 0;
      int rows[4];
      const bool pool_grp = (k0 + 4 * lane) >= nw4 && npool > 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int k = k0 + 4 * lane + e;
        bool valid = false;
        int row;
        if (pool_grp) {
          const int p = k - nw4;
          int w = 0;
          if (k < NK) {
            w = ir ? ir[p] : p;
            valid = w >= 0 && w < vis;
          }
          row = pool_base + (valid ? w : 0);
        } else {
          valid = k < nw;
          const int j = valid ? wlo + (k) : wlo;
          row = win_base + (a.win_ring ? j % a.win_ring : j);
        }
        rows[e] = row;
        if (valid) bits |= 1u << e;
      }
      // gather the 4 bits of every lane into 4 mask words
      uint32_t word = 0;
#pragma unroll
      for (int src = 0; src < 32; ++src) {
        const uint32_t bb = __shfl_sync(0xffffffffu, bits, src);
        if ((src >> 3) == (lane & 3)) word |= bb << ((src & 7) * 4);
      }
      if (lane < 4) ms->mask[lane] = word;
      __syncwarp();
      if (lane == 0) tc::mbar_arrive_expect_tx(&ms->kfull, (uint32_t)(nk * D * 2));
      __syncwarp();
      if (4 * lane < nk) {
        const CUtensorMap* mp = pool_grp ? &map_pool : &map_win;
        uint8_t* dst = smem + L.k + (4 * lane) * 128;
        for (int c = 0; c < nch; ++c)
          tc::tma_gather4(dst + c * 16384, mp, c * 64, rows[0], rows[1], rows[2], rows[3], &ms->kfull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idS = tc::idesc_bf16_f32(128, 64, 0, 0);
    const uint32_t idO = tc::idesc_bf16_f32(128, 64, 1, 1);
    const uint32_t kbase = tc::smem_u32(smem + L.k);
    const uint32_t qbase = tc::smem_u32(smem + L.q);
    const uint32_t pbase = tc::smem_u32(smem + L.p);
    for (int i = 0; i < ntiles; ++i) {
      if (!__all_sync(0xffffffffu, tc::mbar_wait(&ms->kfull, i & 1, kWaitLimit))) {
        if (lane == 0) set_error(ms, 2);
        break;
      }
      tc::tc_fence_after();
      const int nvalid = min(kTile, NK - i * kTile);
      const int nsteps = (nvalid + 15) / 16;
      if (lane == 0) {
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint64_t ad = tc::sdesc_sw128(kbase + off, 16, 1024);
          const uint64_t bd = tc::sdesc_sw128(qbase + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
          tc::umma_f16(tS, ad, bd, idS, kk > 0 ? 1u : 0u);
        }
        tc::umma_commit(&ms->sfull);
      }
      __syncwarp();
      if (!__all_sync(0xffffffffu, tc::mbar_wait(&ms->pfull, i & 1, kWaitLimit))) {
        if (lane == 0) set_error(ms, 4);
        break;
      }
      tc::tc_fence_after();
      if (lane == 0) {
        for (int j = 0; j < nvt; ++j) {
          for (int kk = 0; kk < nsteps; ++kk) {
            const uint64_t ad = tc::sdesc_sw128(kbase + (2 * j) * 16384 + kk * 2048, 16384, 1024);
            const uint64_t bd = tc::sdesc_sw128(pbase + kk * 2048, 16384, 1024);
            tc::umma_f16(tO + 64 * j, ad, bd, idO, (i > 0 || kk > 0) ? 1u : 0u);
          }
        }
        tc::umma_commit(&ms->odone);
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int q4 = warp & 3;                  // TMEM lane quadrant of this warp
    const int kk = q4 * 32 + lane;            // key of the tile owned by this thread
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const float c1 = a.scale * kLog2e;
    float l[kH];
#pragma unroll
    for (int h = 0; h < kH; ++h) l[h] = 0.f;
    float sv[kH];
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
      // the 128 softmax threads leave together or not at all (named barriers follow)
      if (!tc::named_bar_and(1, 128, tc::mbar_wait(&ms->sfull, i & 1, kWaitLimit))) {
        if (kk == 0) set_error(ms, 5);
        ok = false;
        break;
      }
      tc::tc_fence_after();
      tc::tmem_ld_x64(tS + lane_off, sv);
      const bool valid = (ms->mask[kk >> 5] >> (kk & 31)) & 1u;
      bool need = false;
#pragma unroll
      for (int h = 0; h < kH; ++h) {
        sv[h] *= c1;
        need |= valid && (sv[h] - ms->m[h] > kRescaleThreshold);
      }
      if (__any_sync(0xffffffffu, need) && lane == 0) atomicAdd(&ms->rescale_cnt[i & 1], 1);
      tc::named_bar_sync(1, 128);
      const bool rescale = ms->rescale_cnt[i & 1] != 0;
      if (tid == kSoftmaxWarp0 * 32) ms->rescale_cnt[(i + 1) & 1] = 0;
      if (rescale) {
        // tile max per head over the 128 keys, then raise the running max
#pragma unroll
        for (int h = 0; h < kH; ++h) {
          float v = valid ? sv[h] : -INFINITY;
          v = warp_max(v);
          if (lane == 0) ms->red[q4][h] = v;
        }
        tc::named_bar_sync(1, 128);
        if (tid < kSoftmaxWarp0 * 32 + kH) {
          const int h = tid - kSoftmaxWarp0 * 32;
          const float tm = fmaxf(fmaxf(ms->red[0][h], ms->red[1][h]), fmaxf(ms->red[2][h], ms->red[3][h]));
          const float mo = ms->m[h];
          const float mn = fmaxf(mo, tm);
          ms->fac[h] = tc::ex2(mo - mn);
          ms->m[h] = mn;
        }
        tc::named_bar_sync(1, 128);
#pragma unroll
        for (int h = 0; h < kH; ++h) l[h] *= ms->fac[h];
        if (i > 0) {  // O^T holds tiles 0..i-1 (PV(i-1) completed before this tile was loaded)
          float o[kH];
          for (int j = 0; j < nvt; ++j) {
            tc::tmem_ld_x64(tO + 64 * j + lane_off, o);
#pragma unroll
            for (int h = 0; h < kH; ++h) o[h] *= ms->fac[h];
            tc::tmem_st_x64(tO + 64 * j + lane_off, o);
          }
        }
        tc::named_bar_sync(1, 128);
      }
      // probabilities -> P^T row `kk` (bf16, 128B-swizzled MN-major B operand)
      uint8_t* prow = smem + L.p + kk * 128;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int h = u * 8 + 2 * e;
          const float p0 = valid ? tc::ex2(sv[h] - ms->m[h]) : 0.f;
          const float p1 = valid ? tc::ex2(sv[h + 1] - ms->m[h + 1]) : 0.f;
          l[h] += p0;
          l[h + 1] += p1;
          __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
          w4[e] = *reinterpret_cast<uint32_t*>(&pr);
        }
        *reinterpret_cast<uint4*>(prow + ((u ^ (kk & 7)) * 16)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      tc::mbar_arrive(&ms->pfull);
    }

    // ------------------------------------------------------------ epilogue
    const bool have = ok && ntiles > 0;
    if (have && !tc::mbar_wait(&ms->odone, (ntiles - 1) & 1, kWaitLimit)) set_error(ms, 6);
    tc::tc_fence_after();
    // denominators: per-thread partials -> shared memory (the K tile is free now) -> per head
    float* lpart = reinterpret_cast<float*>(smem + L.k);  // [128][65], 33 KB
#pragma unroll
    for (int h = 0; h < kH; ++h) lpart[kk * 65 + h] = l[h];
    tc::named_bar_sync(1, 128);
    if (kk < kH) {
      float sum = 0.f;
      for (int r = 0; r < 128; ++r) sum += lpart[r * 65 + kk];
      const float sink2 = a.sink[kk] * kLog2e;
      ms->inv_l[kk] = 1.f / (sum + tc::ex2(sink2 - ms->m[kk]));
    }
    tc::named_bar_sync(1, 128);
    __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(smem + L.k + 36864);  // [64][dv]
    const int rope_lo = D - R;
    for (int j = 0; j < nvt; ++j) {
      float o[kH];
      if (have) {
        tc::tmem_ld_x64(tO + 64 * j + lane_off, o);
        } else {
#pragma unroll
        for (int h = 0; h < kH; ++h) o[h] = 0.f;
      }
      const int d = 128 * j + kk;
      const bool rot = a.rotate_out && d >= rope_lo;
      float c = 1.f, sn = 0.f;
      if (rot) {
        c = ms->cs[(d - rope_lo) >> 1];
        sn = ms->sn[(d - rope_lo) >> 1];
      }
#pragma unroll
      for (int h = 0; h < kH; ++h) {
        float v = o[h] * ms->inv_l[h];
        const float other = __shfl_xor_sync(0xffffffffu, v, 1);
        if (rot) v = (d & 1) == 0 ? v * c + other * sn : v * c - other * sn;
        stage[h * a.dv + d] = __float2bfloat16_rn(v);
      }
    }
    tc::named_bar_sync(1, 128);
    uint4* og = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + qrow * kH * a.dv);
    const uint4* sg = reinterpret_cast<const uint4*>(stage);
    for (int i = kk; i < kH * a.dv / 8; i += 128) og[i] = sg[i];
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

// Rows of D bf16 values; boxes of 64 columns x 1 row with the 128-byte swizzle.
bool make_row_map(CUtensorMap* m, const void* base, int D, int64_t rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows < 1) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, 1};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

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

bool attn_tc_supported(const AttnArgs& a, int dtype) {
  if (dtype != DSV4_BF16 || a.H != kH) return false;
  if (a.D % 64 != 0 || a.D < 128 || a.D > 576) return false;
  if (a.dv % 128 != 0 || a.dv > 512 || a.dv > a.D) return false;
  if (a.D > 512 && a.dv > a.D - 64) return false;
  if (a.R > 128 || ((a.D - a.R) % 8) != 0) return false;
  if (!a.pool && a.P_cap > 0) return false;
  // the epilogue stages the denominators (33 KB) and the output tile in the free K tile
  if ((a.D / 64) * 16384 < 36864 + 128 * a.dv) return false;
  return encode_fn() != nullptr;
}

cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t st) {
  const int64_t rows = (int64_t)a.B * a.Sq;
  if (rows == 0) return cudaSuccess;
  CUtensorMap mw, mp;
  const int64_t pool_rows = (int64_t)a.B * (a.P_cap > 0 ? a.P_cap : 1);
  const void* pool_ptr = a.pool ? a.pool : a.kv_win;
  if (!make_row_map(&mp, pool_ptr, a.D, pool_rows)) return cudaErrorInvalidValue;
  if (a.n_win > 0 && a.kv_win) {
    const int64_t wr = (int64_t)a.B * (a.win_ring ? a.win_ring : a.kv_rows);
    if (!make_row_map(&mw, a.kv_win, a.D, wr)) return cudaErrorInvalidValue;
  } else {
    mw = mp;  // no window branch: never read
  }
  const Smem L = smem_layout(a.D);
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (e != cudaSuccess) return e;
  attn_tc_kernel<<<(unsigned)rows, kThreads, L.total, st>>>(mw, mp, a);
  note_launch();
  return cudaGetLastError();
}

}  // namespace dsv4
