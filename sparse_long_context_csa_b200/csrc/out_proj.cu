// Grouped low-rank output projection on the sm_100a tensor cores (tcgen05 + TMEM, TMA-fed).
//
// Method: "DeepSeek-V4" doc, "Hybrid attention (§2.3)", the grouped output projection bullet
// (o_groups head groups -> o_lora_rank per group -> hidden_size: DeepseekV4GroupedLinear
// `o_a_proj`, then `o_b_proj`; attention_bias False).  Group i holds the contiguous heads
// [i*H/g, (i+1)*H/g); their outputs, concatenated in head order, are one row of K = (H/g)*dv
// channels, which is exactly columns [i*K, (i+1)*K) of the attention output viewed as a
// [T, H*dv] matrix.  So both projections are "TN" products with K-contiguous operands:
//   u[:, i*dg:(i+1)*dg] = o[:, i*K:(i+1)*K] . wa[i]^T      (g products, K = (H/g)*dv)
//   y                   = u . wb^T                          (one product, K = g*dg)
// u is kept in bf16 between the two launches (the activation dtype of the layer).
//
// Design (one kernel for both products): a persistent CTA per SM walks 128 x 256 output
// tiles (group-major, then row tiles, then column tiles, round-robin over CTAs).
//  * warp 0: TMA producer.  A 128 x 64 box of the left operand and a 256 x 64 box of the
//    right operand per stage (16 KB + 32 KB, 128-byte swizzle), four stages.
//  * warp 1: TMEM owner and MMA issuer: four M=128, N=256, K=16 bf16 MMAs per stage into
//    one of two TMEM accumulators (2 x 256 columns), so the epilogue of a tile overlaps the
//    main loop of the next one.
//  * warps 2-5: epilogue, one TMEM lane quadrant each (thread = output row): 32-column TMEM
//    loads, bf16 conversion, 16-byte stores of the row's 64-byte pieces.
// Rows past T read zeros (TMA fill) and are not stored.  Every wait is bounded; a role that
// gives up records g_out_proj_error and leaves, and the others time out behind it.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "tc_ptx.cuh"

namespace dsv4 {

__device__ int g_out_proj_error = 0;

namespace {

constexpr int kBM = 128, kBN = 256, kBK = 64, kStages = 4;
constexpr int kThreads = 192;
constexpr uint32_t kStageA = kBM * kBK * 2, kStageB = kBN * kBK * 2;  // 16 KB, 32 KB
constexpr uint32_t kSmemData = kStages * (kStageA + kStageB);
constexpr uint32_t kSmemTotal = kSmemData + 1024;                    // + barriers
constexpr uint32_t kWaitLimit = 1u << 22;

struct GemmParams {
  int M;            // rows (tokens)
  int N;            // output columns of one group
  int K;            // reduction length of one group
  int groups;
  int64_t ldc;      // elements between rows of C
  __nv_bfloat16* C;
  int a_col0_step;  // A column offset between groups (= K for o_a_proj, 0 otherwise)
  int b_row0_step;  // B row offset between groups (= N)
  int64_t c_col0_step;
};

struct Bars {
  uint64_t full[kStages], empty[kStages], acc_full[2], acc_empty[2];
  uint32_t tmem_base;
};

__device__ __forceinline__ bool wait_ok(uint64_t* bar, uint32_t parity) {
  return tc::mbar_wait(bar, parity, kWaitLimit);
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_tn_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                   const __grid_constant__ GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((tc::smem_u32(smem) & 1023u) != 0) {
    if (tid == 0) atomicExch(&g_out_proj_error, 3);
    return;
  }
  Bars* bars = reinterpret_cast<Bars*>(smem + kSmemData);
  const int m_tiles = (p.M + kBM - 1) / kBM, n_tiles = p.N / kBN, k_steps = p.K / kBK;
  const int64_t tiles = (int64_t)p.groups * m_tiles * n_tiles;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&bars->full[s], 1);
      tc::mbar_init(&bars->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&bars->acc_full[b], 1);
      tc::mbar_init(&bars->acc_empty[b], 4);  // one arrival per epilogue warp
    }
    tc::mbar_fence_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(&bars->tmem_base, 512);
    tc::tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tc::prefetch_tensormap(&map_a);
    tc::prefetch_tensormap(&map_b);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        const int nt = (int)(t % n_tiles);
        const int mt = (int)((t / n_tiles) % m_tiles);
        const int grp = (int)(t / ((int64_t)n_tiles * m_tiles));
        const int a_x0 = grp * p.a_col0_step, b_y = grp * p.b_row0_step + nt * kBN, a_y = mt * kBM;
        for (int k = 0; k < k_steps; ++k, ++it) {
          const int s = (int)(it % kStages);
          if (it >= kStages && !wait_ok(&bars->empty[s], ((it / kStages) - 1) & 1)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * (kStageA + kStageB);
          tc::mbar_arrive_expect_tx(&bars->full[s], kStageA + kStageB);
          tc::tma_load_2d(sa, &map_a, a_x0 + k * kBK, a_y, &bars->full[s]);
          tc::tma_load_2d(sa + kStageA, &map_b, k * kBK, b_y, &bars->full[s]);
        }
      }
      if (!ok) atomicExch(&g_out_proj_error, 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    const uint32_t idesc = tc::idesc_bf16_f32(kBM, kBN, 0, 0);
    uint32_t it = 0, lt = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++lt) {
      const int buf = (int)(lt & 1);
      if (lt >= 2 && !__all_sync(0xffffffffu, wait_ok(&bars->acc_empty[buf], ((lt >> 1) - 1) & 1))) {
        ok = false;
        break;
      }
      tc::tc_fence_after();
      const uint32_t acc = tmem + buf * kBN;
      for (int k = 0; k < k_steps; ++k, ++it) {
        const int s = (int)(it % kStages);
        if (!__all_sync(0xffffffffu, wait_ok(&bars->full[s], (it / kStages) & 1))) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        if (lane == 0) {
          const uint32_t a0 = tc::smem_u32(smem + s * (kStageA + kStageB));
          const uint32_t b0 = a0 + kStageA;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = tc::sdesc_sw128(a0 + kk * 32, 16, 1024);
            const uint64_t bd = tc::sdesc_sw128(b0 + kk * 32, 16, 1024);
            tc::umma_f16(acc, ad, bd, idesc, (k > 0 || kk > 0) ? 1u : 0u);
          }
          tc::umma_commit(&bars->empty[s]);  // the stage is free once these MMAs have read it
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) tc::umma_commit(&bars->acc_full[buf]);
      __syncwarp();
    }
    if (!ok && lane == 0) atomicExch(&g_out_proj_error, 2);
  } else {
    // ------------------------------------------------------------------ epilogue
    const int q4 = warp & 3;  // TMEM lane quadrant this warp may access
    const int row = q4 * 32 + lane;
    uint32_t lt = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++lt) {
      const int nt = (int)(t % n_tiles);
      const int mt = (int)((t / n_tiles) % m_tiles);
      const int grp = (int)(t / ((int64_t)n_tiles * m_tiles));
      const int buf = (int)(lt & 1);
      if (!__all_sync(0xffffffffu, wait_ok(&bars->acc_full[buf], (lt >> 1) & 1))) {
        ok = false;
        break;
      }
      tc::tc_fence_after();
      const int m = mt * kBM + row;
      __nv_bfloat16* crow = p.C + (int64_t)m * p.ldc + grp * p.c_col0_step + (int64_t)nt * kBN;
      const uint32_t acc = tmem + buf * kBN + ((uint32_t)(q4 * 32) << 16);
#pragma unroll 1
      for (int j = 0; j < kBN / 32; ++j) {
        float v[32];
        tc::tmem_ld_x32(acc + j * 32, v);
        if (m < p.M) {
          uint4 pk[4];
          uint32_t* w = reinterpret_cast<uint32_t*>(pk);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
            w[e] = *reinterpret_cast<uint32_t*>(&b2);
          }
          uint4* dst = reinterpret_cast<uint4*>(crow + j * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = pk[e];
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bars->acc_empty[buf]);
    }
    if (!ok && lane == 0) atomicExch(&g_out_proj_error, 4);
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
    void* q = nullptr;
    cudaDriverEntryPointQueryResult r;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &q, cudaEnableDefault, &r) == cudaSuccess &&
        r == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(q);
  }
  return fn;
}

// A [rows, cols] bf16 matrix with row stride ld elements; boxes of 64 columns x box_rows rows,
// 128-byte swizzle; reads past the last row return zeros.
bool make_map(CUtensorMap* m, const void* base, int64_t cols, int64_t rows, int64_t ld, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows < 1 || cols < 1) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// C[:, grp*c_step + n] = sum_k A[:, grp*a_step + k] B[grp*N + n, k] for every group.
cudaError_t launch_gemm(const void* A, int64_t a_cols, int64_t lda, const void* B, int64_t b_rows, int64_t ldb,
                        GemmParams p, cudaStream_t st) {
  CUtensorMap ma, mb;
  if (!make_map(&ma, A, a_cols, p.M, lda, kBM)) return cudaErrorInvalidValue;
  if (!make_map(&mb, B, p.K, b_rows, ldb, kBN)) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(gemm_tn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemTotal);
  if (e != cudaSuccess) return e;
  const int64_t tiles = (int64_t)p.groups * ((p.M + kBM - 1) / kBM) * (p.N / kBN);
  const int nsm = sm_count();
  const int grid = (int)(tiles < nsm ? tiles : nsm);
  gemm_tn_kernel<<<grid, kThreads, kSmemTotal, st>>>(ma, mb, p);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

bool out_proj_supported(const OutProjArgs& a) {
  const int64_t width = (int64_t)(a.H / a.groups) * a.dv;  // channels of one head group
  return a.groups >= 1 && a.H % a.groups == 0 && width % kBK == 0 && a.dg % kBN == 0 &&
         ((int64_t)a.groups * a.dg) % kBK == 0 && a.hidden % kBN == 0 && encode_fn() != nullptr;
}

cudaError_t launch_out_proj(const OutProjArgs& a, cudaStream_t st) {
  if (a.T == 0) return cudaSuccess;
  const int64_t width = (int64_t)(a.H / a.groups) * a.dv;
  const int64_t inner = (int64_t)a.groups * a.dg;
  GemmParams pa{};  // u = grouped o_a_proj(o)
  pa.M = a.T;
  pa.N = a.dg;
  pa.K = (int)width;
  pa.groups = a.groups;
  pa.ldc = inner;
  pa.C = static_cast<__nv_bfloat16*>(a.u);
  pa.a_col0_step = (int)width;
  pa.b_row0_step = a.dg;
  pa.c_col0_step = a.dg;
  cudaError_t e = launch_gemm(a.o, (int64_t)a.H * a.dv, (int64_t)a.H * a.dv, a.wa, inner, width, pa, st);
  if (e != cudaSuccess) return e;
  GemmParams pb{};  // y = o_b_proj(u)
  pb.M = a.T;
  pb.N = a.hidden;
  pb.K = (int)inner;
  pb.groups = 1;
  pb.ldc = a.hidden;
  pb.C = static_cast<__nv_bfloat16*>(a.y);
  return launch_gemm(a.u, inner, inner, a.wb, a.hidden, inner, pb, st);
}

cudaError_t take_out_proj_error(int* code) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_out_proj_error, sizeof(int));
  if (e != cudaSuccess) return e;
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_out_proj_error, &zero, sizeof(int));
  }
  *code = v;
  return e;
}

}  // namespace dsv4
