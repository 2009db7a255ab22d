// KV compressor: softmax-gated per-channel pooling of token rows into pool entries,
// with RoPE on the entry's trailing channels; also writes the rotated token rows
// (the sliding-window keys) in the same pass over x.
//
// Method: "DeepSeek-V4" doc, "Hybrid attention (§2.3)" — CSA pools with overlapping
// windows at m=4, HCA with non-overlapping windows at m'=128; "Cache layers" — the
// indexer keys are pooled the same way at index_head_dim.
//
// One CTA per token block w (tokens [wm, (w+1)m)) and sequence b.  Each thread owns a
// channel pair (d, d+1) so that a RoPE pair never crosses threads; a warp reads 32
// consecutive pairs of a row (128 B of bf16, 256 B of fp32), so every row is read
// coalesced.  The softmax over the window is an online (running max) softmax in fp32.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace dsv4 {

template <typename T>
__global__ void __launch_bounds__(256) compress_kernel(CompressArgs a) {
  const int w = blockIdx.x;
  const int b = blockIdx.y;
  const int c = a.c;
  const int S = a.S;
  const int m = a.m;
  const int P = S / m;
  const T* __restrict__ x = static_cast<const T*>(a.x) + (int64_t)b * S * c;
  const T* __restrict__ z = a.z ? static_cast<const T*>(a.z) + (int64_t)b * S * c : nullptr;
  const int64_t* pos = a.pos ? a.pos + (int64_t)b * S : nullptr;
  const int rope_lo = c - a.R;

  if (w < P) {
    const int lo = a.overlap ? (w - 1) * m : w * m;
    const int hi = (w + 1) * m;
    const int j0 = lo < 0 ? 0 : lo;
    T* __restrict__ pool = static_cast<T*>(a.pool) + ((int64_t)b * a.P_cap + w) * c;
    for (int pr = threadIdx.x; pr < c / 2; pr += blockDim.x) {
      const int d = 2 * pr;
      float mx0 = -INFINITY, mx1 = -INFINITY, s0 = 0.f, s1 = 0.f, acc0 = 0.f, acc1 = 0.f;
#pragma unroll 4
      for (int j = j0; j < hi; ++j) {
        const float2 xv = load2<T>(x + (int64_t)j * c + d);
        float l0 = 0.f, l1 = 0.f;
        if (z) {
          const float2 zv = load2<T>(z + (int64_t)j * c + d);
          l0 = zv.x;
          l1 = zv.y;
        }
        if (a.bias) {
          const float2 bv = *reinterpret_cast<const float2*>(a.bias + (int64_t)(j - lo) * c + d);
          l0 += bv.x;
          l1 += bv.y;
        }
        if (l0 > mx0) {
          const float r = expf(mx0 - l0);
          s0 *= r;
          acc0 *= r;
          mx0 = l0;
        }
        if (l1 > mx1) {
          const float r = expf(mx1 - l1);
          s1 *= r;
          acc1 *= r;
          mx1 = l1;
        }
        const float e0 = expf(l0 - mx0), e1 = expf(l1 - mx1);
        s0 += e0;
        s1 += e1;
        acc0 = fmaf(e0, xv.x, acc0);
        acc1 = fmaf(e1, xv.y, acc1);
      }
      float v0 = acc0 / s0, v1 = acc1 / s1;
      if (a.apply_rope && d >= rope_lo) {
        float cs, sn;
        rope_cos_sin(pos[(int64_t)w * m], (d - rope_lo) / 2, a.R, a.theta, &cs, &sn);
        const float r0 = v0 * cs - v1 * sn;
        const float r1 = v0 * sn + v1 * cs;
        v0 = r0;
        v1 = r1;
      }
      store2<T>(pool + d, v0, v1);
    }
  }

  if (a.x_rot) {
    T* __restrict__ xr = static_cast<T*>(a.x_rot) + (int64_t)b * S * c;
    const int t_hi = min((w + 1) * m, S);
    const int npairs = c / 2;
    for (int it = threadIdx.x; it < (t_hi - w * m) * npairs; it += blockDim.x) {
      const int j = w * m + it / npairs;
      const int d = 2 * (it % npairs);
      float2 v = load2<T>(x + (int64_t)j * c + d);
      if (d >= rope_lo) {
        float cs, sn;
        rope_cos_sin(pos[j], (d - rope_lo) / 2, a.R, a.theta, &cs, &sn);
        const float r0 = v.x * cs - v.y * sn;
        const float r1 = v.x * sn + v.y * cs;
        v = make_float2(r0, r1);
      }
      store2<T>(xr + (int64_t)j * c + d, v.x, v.y);
    }
  }
}

cudaError_t launch_compress(const CompressArgs& a, int dtype, cudaStream_t st) {
  const int nblk = (a.S + a.m - 1) / a.m;
  if (nblk == 0 || a.B == 0) return cudaSuccess;
  int threads = ((a.c / 2 + 31) / 32) * 32;
  threads = threads < 32 ? 32 : (threads > 256 ? 256 : threads);
  dim3 grid(nblk, a.B);
  if (dtype == DSV4_BF16)
    compress_kernel<__nv_bfloat16><<<grid, threads, 0, st>>>(a);
  else
    compress_kernel<float><<<grid, threads, 0, st>>>(a);
  note_launch();
  return cudaGetLastError();
}

}  // namespace dsv4
