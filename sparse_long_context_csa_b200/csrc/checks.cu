// Optional device-side validation of the attention's index lists.
//
// Method: "DeepSeek-V4" doc, "Attention mask layout" — query t sees pool entry w only once
// the entry's window has closed (w < (t+1)/m); empty top-k slots hold the -1 sentinel; each
// selected entry is one key of the query.  The attention kernels never read out of bounds on
// a bad list (an entry that is not visible is masked and its gather is redirected to row 0),
// but they would silently drop an out-of-range entry or count a duplicated one twice.  With
// the checks on, every list is validated first and a violation sets an error word that
// dsv4_device_check reports; nothing traps.
//
// One CTA per query row: the row's visible entries are a bitmap in shared memory; a thread
// that finds its entry's bit already set has found a duplicate.
#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace dsv4 {

__device__ int g_index_check_error = 0;  // bit 0: entry out of range / not visible; bit 1: duplicate

namespace {

#ifdef DSV4_DEBUG
std::atomic<int> g_checks_on{1};
#else
std::atomic<int> g_checks_on{0};
#endif

constexpr int kCheckThreads = 256;
// 192 KB of shared memory: duplicates are detected in rows of up to 1,572,864 visible entries
// (longer rows get the range check only)
constexpr int kMaxBitmapWords = 48 * 1024;

__global__ void __launch_bounds__(kCheckThreads) index_check_kernel(const int32_t* __restrict__ idx,
                                                                    const int32_t* __restrict__ q_index, int Sq,
                                                                    int topk, int m, int P_cap) {
  extern __shared__ uint32_t seen[];
  const int64_t row = blockIdx.x;
  const int t = query_cache_index(q_index, row, (int)(row % Sq));
  const int vis = visible_entries(t, m, P_cap);
  const int words = (vis + 31) / 32;
  const bool bitmap = words <= kMaxBitmapWords;
  if (bitmap)
    for (int i = threadIdx.x; i < words; i += kCheckThreads) seen[i] = 0u;
  __syncthreads();
  int bad = 0;
  const int32_t* ir = idx + row * topk;
  for (int k = threadIdx.x; k < topk; k += kCheckThreads) {
    const int w = ir[k];
    if (w == -1) continue;
    if (w < 0 || w >= vis) {
      bad |= 1;
      continue;
    }
    if (bitmap) {
      const uint32_t bit = 1u << (w & 31);
      if (atomicOr(&seen[w >> 5], bit) & bit) bad |= 2;
    }
  }
  if (bad) atomicOr(&g_index_check_error, bad);
}

}  // namespace

void set_index_checks(int on) { g_checks_on.store(on ? 1 : 0); }
bool index_checks_on() { return g_checks_on.load() != 0; }

cudaError_t launch_index_check(const int32_t* idx, const int32_t* q_index, int64_t rows, int Sq, int topk, int m,
                               int P_cap, cudaStream_t st) {
  if (rows == 0 || topk < 1) return cudaSuccess;
  const int words = (P_cap + 31) / 32;
  const size_t smem = (size_t)(words < kMaxBitmapWords ? words : kMaxBitmapWords) * sizeof(uint32_t);
  cudaError_t e = cudaFuncSetAttribute(index_check_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  index_check_kernel<<<(unsigned)rows, kCheckThreads, smem, st>>>(idx, q_index, Sq, topk, m, P_cap);
  note_launch();
  return cudaGetLastError();
}

cudaError_t take_index_check_error(int* code) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_index_check_error, sizeof(int));
  if (e != cudaSuccess) return e;
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_index_check_error, &zero, sizeof(int));
  }
  *code = v;
  return e;
}

}  // namespace dsv4
