// Sparse shared-K=V MQA attention with sink on CUDA cores, exact fp32 arithmetic.
//
// Method: "DeepSeek-V4" doc, "Hybrid attention (§2.3)" — single K=V head read as key
// and value, partial interleaved RoPE on the trailing channels with the -i rotation of
// the output rope slice (eq. 26), per-head learnable sink (eq. 27), and the
// sliding-window K=V rows concatenated with the compressor entries before the core
// attention; "Attention mask layout" — -1 slots select nothing.
//
// This is the reference-precision path (fp32 workloads and shapes the tensor-core kernel
// does not cover).  One CTA per (query, group of 8 heads); warp = head.  Key rows are
// staged 32 at a time in shared memory as fp32 and shared by the 8 heads (MQA); lane l
// scores key l, the online softmax runs across the warp, and each lane accumulates
// dv/32 output channels.  The sink enters as the initial running max / denominator
// (an extra logit whose value row is zero).
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dsv4 {

namespace {

constexpr int kHeadsPerCta = 8;
constexpr int kKeysPerChunk = 32;
constexpr int kMaxDvPerLane = 18;  // dv <= 576

// Key slot i of query (b,s): window rows first, then the idx slots.
// Returns a row pointer into kv_win / pool, or nullptr for an empty slot.
template <typename T>
__device__ __forceinline__ const T* key_row(const AttnArgs& a, int b, int64_t qrow, int t, int nwin_keys,
                                            int wlo, int vis, int i) {
  if (i < nwin_keys) {
    const int j = wlo + i;
    const int64_t slot = a.win_ring ? (int64_t)(j % a.win_ring) : (int64_t)j;
    const int64_t rows = a.win_ring ? a.win_ring : a.kv_rows;
    if (slot >= rows) return nullptr;  // a cache index past the window buffer selects nothing
    return static_cast<const T*>(a.kv_win) + ((int64_t)b * rows + slot) * a.D;
  }
  const int k = i - nwin_keys;
  int w;
  if (a.idx) {
    w = a.idx[qrow * a.topk + k];
    if (w < 0 || w >= vis) return nullptr;  // empty slot (or an entry not yet visible)
  } else {
    w = k;
  }
  return static_cast<const T*>(a.pool) + ((int64_t)b * a.P_cap + w) * a.D;
}

template <typename T>
__global__ void __launch_bounds__(256) attn_simt_kernel(AttnArgs a) {
  extern __shared__ float sm[];
  const int D = a.D;
  float* qs = sm;                                   // [8][D]
  float* ks = qs + kHeadsPerCta * D;                // [32][D+1]
  __shared__ const void* rowp[kKeysPerChunk];

  const int64_t qrow = blockIdx.x;  // b*Sq + s
  const int b = (int)(qrow / a.Sq);
  const int s = (int)(qrow % a.Sq);
  const int h0 = blockIdx.y * kHeadsPerCta;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = h0 + warp;

  const int t = query_cache_index(a.q_index, qrow, s);
  const int vis = visible_entries(t, a.m, a.P_cap);
  const int wlo = t - a.n_win + 1 > 0 ? t - a.n_win + 1 : 0;
  const int nwin_keys = a.n_win > 0 ? t - wlo + 1 : 0;
  const int npool_slots = a.idx ? a.topk : vis;
  const int nslots = nwin_keys + npool_slots;

  // q rows of the CTA's heads, rotated at qpos when asked
  const T* q = static_cast<const T*>(a.q);
  const int rope_lo = D - a.R;
  for (int i = threadIdx.x; i < kHeadsPerCta * D / 2; i += blockDim.x) {
    const int hh = (2 * i) / D, d = (2 * i) % D;
    float2 v = make_float2(0.f, 0.f);
    if (h0 + hh < a.H) {
      v = load2<T>(q + (qrow * a.H + h0 + hh) * D + d);
      if (a.rope_q && d >= rope_lo) {
        float cs, sn;
        rope_cos_sin(a.qpos[qrow], (d - rope_lo) / 2, a.R, a.theta, &cs, &sn);
        v = make_float2(v.x * cs - v.y * sn, v.x * sn + v.y * cs);
      }
    }
    qs[hh * D + d] = v.x;
    qs[hh * D + d + 1] = v.y;
  }

  const float sink = h < a.H ? a.sink[h] : 0.f;
  float mx = sink, den = 1.f;  // the sink's own term e^{sink - mx}
  float acc[kMaxDvPerLane];
#pragma unroll
  for (int i = 0; i < kMaxDvPerLane; ++i) acc[i] = 0.f;
  const int nv = a.dv / 32;

  for (int base = 0; base < nslots; base += kKeysPerChunk) {
    __syncthreads();
    if (threadIdx.x < kKeysPerChunk) {
      const int i = base + threadIdx.x;
      rowp[threadIdx.x] = i < nslots ? (const void*)key_row<T>(a, b, qrow, t, nwin_keys, wlo, vis, i) : nullptr;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kKeysPerChunk * D / 2; i += blockDim.x) {
      const int r = (2 * i) / D, d = (2 * i) % D;
      const T* p = static_cast<const T*>(rowp[r]);
      const float2 v = p ? load2<T>(p + d) : make_float2(0.f, 0.f);
      ks[r * (D + 1) + d] = v.x;
      ks[r * (D + 1) + d + 1] = v.y;
    }
    __syncthreads();
    if (h >= a.H) continue;

    // lane scores key `lane` of the chunk
    float l = -INFINITY;
    if (rowp[lane] != nullptr) {
      const float* kr = ks + lane * (D + 1);
      const float* qr = qs + warp * D;
      float dot = 0.f;
      for (int d = 0; d < D; ++d) dot = fmaf(qr[d], kr[d], dot);
      l = a.scale * dot;
    }
    const float cmax = warp_max(l);
    const float mnew = fmaxf(mx, cmax);
    const float corr = expf(mx - mnew);
    const float p = rowp[lane] != nullptr ? expf(l - mnew) : 0.f;
    den = den * corr + warp_sum(p);
    mx = mnew;
#pragma unroll
    for (int i = 0; i < kMaxDvPerLane; ++i) acc[i] *= corr;
    for (int j = 0; j < kKeysPerChunk; ++j) {
      const float pj = __shfl_sync(0xffffffffu, p, j);
      if (pj == 0.f) continue;
      const float* kr = ks + j * (D + 1);
#pragma unroll
      for (int i = 0; i < kMaxDvPerLane; ++i)
        if (i < nv) acc[i] = fmaf(pj, kr[lane + 32 * i], acc[i]);
    }
  }
  if (h >= a.H) return;

  const float inv = 1.f / den;
  T* out = static_cast<T*>(a.out) + (qrow * a.H + h) * a.dv;
#pragma unroll
  for (int i = 0; i < kMaxDvPerLane; ++i) {
    if (i >= nv) break;
    const int d = lane + 32 * i;
    float v = acc[i] * inv;
    // -qpos rotation of the rope slice (eq. 26): pair (d, d^1) lives in lanes (lane, lane^1)
    const float other = __shfl_xor_sync(0xffffffffu, v, 1);
    if (a.rotate_out && d >= rope_lo) {
      float cs, sn;
      rope_cos_sin(a.qpos[qrow], (d - rope_lo) / 2, a.R, a.theta, &cs, &sn);
      v = (d & 1) == 0 ? v * cs + other * sn : v * cs - other * sn;
    }
    out[d] = from_f32<T>(v);
  }
}

}  // namespace

cudaError_t launch_attn_simt(const AttnArgs& a, int dtype, cudaStream_t st) {
  const int64_t rows = (int64_t)a.B * a.Sq;
  if (rows == 0) return cudaSuccess;
  const size_t smem = (size_t)(kHeadsPerCta * a.D + kKeysPerChunk * (a.D + 1)) * sizeof(float);
  dim3 grid((unsigned)rows, (a.H + kHeadsPerCta - 1) / kHeadsPerCta);
  if (dtype == DSV4_BF16) {
    cudaFuncSetAttribute(attn_simt_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    attn_simt_kernel<__nv_bfloat16><<<grid, 256, smem, st>>>(a);
  } else {
    cudaFuncSetAttribute(attn_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    attn_simt_kernel<float><<<grid, 256, smem, st>>>(a);
  }
  note_launch();
  return cudaGetLastError();
}

}  // namespace dsv4
