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

// Softmax-gated pooling of channel pair (d, d+1) over tokens j = j0 .. hi-1 of one entry
// window starting at token lo (slot j - lo of the bias); row_of(j) is the row holding token
// j.  An online (running max) softmax in fp32.  Shared by the prefill compressor and the
// decode-cache append, so that both write the same bits for the same rows.
template <typename T, typename RowOf>
__device__ __forceinline__ float2 pool_pair(const T* __restrict__ x, const T* __restrict__ z,
                                            const float* __restrict__ bias, int lo, int j0, int hi, int c, int d,
                                            RowOf row_of) {
  float mx0 = -INFINITY, mx1 = -INFINITY, s0 = 0.f, s1 = 0.f, acc0 = 0.f, acc1 = 0.f;
#pragma unroll 4
  for (int j = j0; j < hi; ++j) {
    const int64_t r = row_of(j);
    const float2 xv = load2<T>(x + r * c + d);
    float l0 = 0.f, l1 = 0.f;
    if (z) {
      const float2 zv = load2<T>(z + r * c + d);
      l0 = zv.x;
      l1 = zv.y;
    }
    if (bias) {
      const float2 bv = *reinterpret_cast<const float2*>(bias + (int64_t)(j - lo) * c + d);
      l0 += bv.x;
      l1 += bv.y;
    }
    if (l0 > mx0) {
      const float q = expf(mx0 - l0);
      s0 *= q;
      acc0 *= q;
      mx0 = l0;
    }
    if (l1 > mx1) {
      const float q = expf(mx1 - l1);
      s1 *= q;
      acc1 *= q;
      mx1 = l1;
    }
    const float e0 = expf(l0 - mx0), e1 = expf(l1 - mx1);
    s0 += e0;
    s1 += e1;
    acc0 = fmaf(e0, xv.x, acc0);
    acc1 = fmaf(e1, xv.y, acc1);
  }
  return make_float2(acc0 / s0, acc1 / s1);
}

// RoPE of channel pair (d, d+1) when it lies in the trailing R channels; inv_freq[k] =
// theta^(-2k/R) comes from the host, the angle pos * inv_freq[k] is formed and reduced to
// [-pi, pi] in double precision (positions up to 2^20 keep full float accuracy), then its
// cos/sin are taken in float.
__device__ __forceinline__ float2 rope_pair(float2 v, int64_t pos, int d, int c, int R, const double* inv_freq) {
  const int rope_lo = c - R;
  if (d < rope_lo) return v;
  double ang = (double)pos * inv_freq[(d - rope_lo) / 2];
  ang -= rint(ang * 0.15915494309189535) * 6.283185307179586;
  float sn, cs;
  sincosf((float)ang, &sn, &cs);
  return make_float2(v.x * cs - v.y * sn, v.x * sn + v.y * cs);
}

// theta^(-2k/R) for k < R/2 (R <= 2 * kMaxRopePairs, checked by the caller).
inline void fill_inv_freq(double* inv, int R, float theta) {
  for (int k = 0; k < kMaxRopePairs; ++k) inv[k] = (R > 0 && k < R / 2) ? pow((double)theta, -2.0 * k / R) : 0.0;
}

template <typename T>
__global__ void __launch_bounds__(256, 5) compress_kernel(const __grid_constant__ CompressArgs a) {
  const int w = blockIdx.x;
  const int b = blockIdx.y;
  const int c = a.c;
  const int S = a.S;
  const int m = a.m;
  const int P = S / m;
  const T* __restrict__ x = static_cast<const T*>(a.x) + (int64_t)b * S * c;
  const T* __restrict__ z = a.z ? static_cast<const T*>(a.z) + (int64_t)b * S * c : nullptr;
  const int64_t* pos = a.pos ? a.pos + (int64_t)b * S : nullptr;

  if (a.pool && w < P) {
    const int lo = a.overlap ? (w - 1) * m : w * m;
    const int hi = (w + 1) * m;
    const int j0 = lo < 0 ? 0 : lo;
    T* __restrict__ pool = static_cast<T*>(a.pool) + ((int64_t)b * a.P_cap + w) * c;
    for (int pr = threadIdx.x; pr < c / 2; pr += blockDim.x) {
      const int d = 2 * pr;
      float2 v = pool_pair<T>(x, z, a.bias, lo, j0, hi, c, d, [](int j) { return (int64_t)j; });
      if (a.apply_rope) v = rope_pair(v, pos[(int64_t)w * m], d, c, a.R, a.inv_freq);
      store2<T>(pool + d, v.x, v.y);
    }
  }

  if (a.x_rot) {
    // the block's rows as one list of pairs: first every row's pairs before the trailing R
    // channels (copied), then every row's R/2 rotated pairs, so that with many rows the
    // rotations are spread over all threads (a thread keeps no fixed pair)
    T* __restrict__ xr = static_cast<T*>(a.x_rot) + (int64_t)b * S * c;
    const int t0 = w * m;
    const int ntok = min((w + 1) * m, S) - t0;
    const int nrp = a.R / 2;
    const int np0 = c / 2 - nrp;
    const int ncopy = ntok * np0;
    for (int it = threadIdx.x; it < ntok * (np0 + nrp); it += blockDim.x) {
      if (it < ncopy) {
        const int64_t j = t0 + it / np0;
        const int d = 2 * (it % np0);
        const float2 v = load2<T>(x + j * c + d);
        store2<T>(xr + j * c + d, v.x, v.y);
      } else {
        const int k = it - ncopy;
        const int64_t j = t0 + k / nrp;
        const int d = 2 * (np0 + k % nrp);
        const float2 v = rope_pair(load2<T>(x + j * c + d), pos[j], d, c, a.R, a.inv_freq);
        store2<T>(xr + j * c + d, v.x, v.y);
      }
    }
  }
}

cudaError_t launch_compress(const CompressArgs& args, int dtype, cudaStream_t st) {
  const int nblk = (args.S + args.m - 1) / args.m;
  if (nblk == 0 || args.B == 0) return cudaSuccess;
  CompressArgs a = args;
  fill_inv_freq(a.inv_freq, a.R, a.theta);
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

// Decode-cache append: one CTA per sequence, thread per channel pair.  The new token goes to
// buffer slot t % Lw (raw row, logits, position) and, rotated, to window-ring slot
// t % win_ring; when it closes a block, the entry of that block is pooled from the buffer.
//
// The kernel is latency-bound (a few hundred bytes per sequence), so it is built around
// memory round trips.  When the buffer fits in shared memory (kStaged: Lw x c rows of x, z
// and the fp32 bias, plus Lw positions), every read the step can need (the cache index, the
// new row, all Lw buffered rows, the bias, the buffered positions) is issued at once, before
// the cache index is known (no address depends on it), into shared memory; the entry is then
// pooled from there: one round trip instead of four.  Otherwise the buffer is pooled in place
// (the buffered positions, written by thread 0, are read after a barrier).  Both paths pool
// with pool_pair, so the entry has the same bits as the one the prefill compressor writes.
template <typename T, bool kStaged>
__global__ void __launch_bounds__(256) decode_append_kernel(const __grid_constant__ DecodeAppendArgs a) {
  extern __shared__ __align__(16) uint8_t sm[];
  const int b = blockIdx.x;
  const int c = a.c, m = a.m;
  const int lw = a.overlap ? 2 * m : m;
  const int t = a.t[b];
  const int64_t pos = a.pos[b];
  const T* __restrict__ xn = static_cast<const T*>(a.x) + (int64_t)b * c;
  const T* __restrict__ zn = a.z ? static_cast<const T*>(a.z) + (int64_t)b * c : nullptr;
  T* __restrict__ bx = static_cast<T*>(a.buf_x) + (int64_t)b * lw * c;
  T* __restrict__ bz = a.buf_z ? static_cast<T*>(a.buf_z) + (int64_t)b * lw * c : nullptr;
  int64_t* __restrict__ bpos = a.buf_pos + (int64_t)b * lw;

  // where the pooling reads the buffer: in place, or the shared-memory copy
  T* px = bx;
  T* pz = bz;
  const float* pb = a.bias;
  int64_t* ppos = bpos;
  if constexpr (kStaged) {
    px = reinterpret_cast<T*>(sm);
    pz = bz ? px + lw * c : nullptr;
    float* sb = reinterpret_cast<float*>(px + 2 * lw * c);
    ppos = reinterpret_cast<int64_t*>(sb + lw * c);
    for (int d = 2 * threadIdx.x; d < c; d += 2 * blockDim.x) {
#pragma unroll 8
      for (int r = 0; r < lw; ++r) {
        const float2 xv = load2<T>(bx + (int64_t)r * c + d);
        store2<T>(px + r * c + d, xv.x, xv.y);
        if (bz) {
          const float2 zv = load2<T>(bz + (int64_t)r * c + d);
          store2<T>(pz + r * c + d, zv.x, zv.y);
        }
        if (a.bias) *reinterpret_cast<float2*>(sb + r * c + d) = *reinterpret_cast<const float2*>(a.bias + r * c + d);
      }
    }
    if (a.bias) pb = sb;
    for (int r = threadIdx.x; r < lw; r += blockDim.x) ppos[r] = bpos[r];
  }

  const int slot = (t < 0 ? 0 : t) % lw;
  for (int d = 2 * threadIdx.x; d < c; d += 2 * blockDim.x) {
    const float2 xv = load2<T>(xn + d);
    const float2 zv = zn ? load2<T>(zn + d) : make_float2(0.f, 0.f);
    if (t < 0) break;  // the sequence is skipped (the same for every thread of the CTA)
    store2<T>(bx + (int64_t)slot * c + d, xv.x, xv.y);
    if (bz) store2<T>(bz + (int64_t)slot * c + d, zv.x, zv.y);
    if constexpr (kStaged) {
      store2<T>(px + slot * c + d, xv.x, xv.y);
      if (bz) store2<T>(pz + slot * c + d, zv.x, zv.y);
    }
    if (a.win) {
      const float2 v = a.apply_rope ? rope_pair(xv, pos, d, c, a.R, a.inv_freq) : xv;
      store2<T>(static_cast<T*>(a.win) + ((int64_t)b * a.win_ring + t % a.win_ring) * c + d, v.x, v.y);
    }
  }
  if (t < 0) return;
  if (threadIdx.x == 0) bpos[slot] = pos;
  // kStaged: the staged positions of other threads; otherwise thread 0's store above
  __syncthreads();
  if ((t + 1) % m != 0) return;
  const int w = (t + 1) / m - 1;
  if (w >= a.P_cap) return;
  const int lo = a.overlap ? (w - 1) * m : w * m;
  const int j0 = lo < 0 ? 0 : lo;
  const int eslot = (w * m) % lw;
  const int64_t epos = eslot == slot ? pos : ppos[eslot];
  T* __restrict__ pool = static_cast<T*>(a.pool) + ((int64_t)b * a.P_cap + w) * c;
  for (int d = 2 * threadIdx.x; d < c; d += 2 * blockDim.x) {
    float2 v = pool_pair<T>(px, pz, pb, lo, j0, t + 1, c, d, [lw](int j) { return (int64_t)(j % lw); });
    if (a.apply_rope) v = rope_pair(v, epos, d, c, a.R, a.inv_freq);
    store2<T>(pool + d, v.x, v.y);
  }
}

// Shared memory of the staged append: Lw rows of x and z (T), of the bias (fp32) and the Lw
// positions.
inline size_t append_stage_bytes(const DecodeAppendArgs& a, size_t elem) {
  const size_t lw = a.overlap ? 2 * (size_t)a.m : (size_t)a.m;
  return lw * (size_t)a.c * (2 * elem + 4) + lw * 8;
}

cudaError_t launch_decode_append(const DecodeAppendArgs& args, int dtype, cudaStream_t st) {
  if (args.B == 0) return cudaSuccess;
  DecodeAppendArgs a = args;
  fill_inv_freq(a.inv_freq, a.R, a.theta);
  int threads = ((a.c / 2 + 31) / 32) * 32;
  threads = threads < 32 ? 32 : (threads > 256 ? 256 : threads);
  const size_t elem = dtype == DSV4_BF16 ? 2 : 4;
  const size_t stage = append_stage_bytes(a, elem);
  const bool staged = stage <= 48 * 1024;  // within the default dynamic shared-memory limit
  if (dtype == DSV4_BF16) {
    if (staged)
      decode_append_kernel<__nv_bfloat16, true><<<a.B, threads, stage, st>>>(a);
    else
      decode_append_kernel<__nv_bfloat16, false><<<a.B, threads, 0, st>>>(a);
  } else {
    if (staged)
      decode_append_kernel<float, true><<<a.B, threads, stage, st>>>(a);
    else
      decode_append_kernel<float, false><<<a.B, threads, 0, st>>>(a);
  }
  note_launch();
  return cudaGetLastError();
}

}  // namespace dsv4
