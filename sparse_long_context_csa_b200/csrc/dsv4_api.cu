// C ABI of libdsv4: host-side validation, workspace layout and kernel dispatch.
// Declarations and the full contract of each entry point are in include/dsv4.h.
#include <stdint.h>
#include <string.h>

#include <atomic>

#include "internal.h"

using namespace dsv4;

namespace dsv4 {
static std::atomic<uint64_t> g_launches{0};
void note_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }
}  // namespace dsv4

namespace {

constexpr size_t kScoresBudget = 256ull << 20;  // fp32 score rows kept per indexer chunk
constexpr int64_t kSplitChunkRows = 65535;       // query rows per launch of the split indexer calls
constexpr size_t kAlign = 256;

inline size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }


// Keys a query attends at most: the window plus the selected (top-k) or all pool entries.
// Only the sizes enter, so the workspace size and the launch agree on the key split.
int64_t attn_keys_estimate(const dsv4_params* p) {
  const int64_t pool = p->topk > 0 ? (p->topk < p->P_cap ? p->topk : p->P_cap) : p->P_cap;
  return (int64_t)(p->n_win > 0 ? p->n_win : 0) + (pool > 0 ? pool : 0);
}

dsv4_status check_common(const dsv4_params* p) {
  if (!p) return DSV4_ERR_ARG;
  if (p->dtype != DSV4_F32 && p->dtype != DSV4_BF16) return DSV4_ERR_DTYPE;
  if (p->B < 0 || p->S < 0 || p->Sq < 0 || p->H < 0 || p->D < 0) return DSV4_ERR_SHAPE;
  if (p->m < 1 || (p->overlap != 0 && p->overlap != 1)) return DSV4_ERR_SHAPE;
  if (p->P_cap < 0) return DSV4_ERR_SHAPE;
  return DSV4_OK;
}

dsv4_status check_rope(const dsv4_params* p) {
  if (p->R < 0 || (p->R & 1) || p->R > p->D) return DSV4_ERR_SHAPE;
  if (!(p->rope_theta > 0.f)) return DSV4_ERR_SHAPE;
  return DSV4_OK;
}

dsv4_status check_indexer(const dsv4_params* p) {
  if (p->nI < 1 || p->nI > 64 || (64 % p->nI) != 0) return DSV4_ERR_SHAPE;
  if (p->cI != 32 && p->cI != 64 && p->cI != 128) return DSV4_ERR_SHAPE;
  if (p->topk < 1 || p->P_cap < 1) return DSV4_ERR_SHAPE;
  return DSV4_OK;
}

dsv4_status check_attn(const dsv4_params* p) {
  if (p->H < 1 || p->D < 2 || (p->D & 1) || p->D > 1024) return DSV4_ERR_SHAPE;
  if (p->dv < 32 || p->dv > p->D || (p->dv % 32) != 0 || p->dv > 576) return DSV4_ERR_SHAPE;
  if (p->n_win < 0 || p->win_ring < 0 || (p->win_ring > 0 && p->win_ring < p->n_win)) return DSV4_ERR_SHAPE;
  if (p->rotate_out && p->dv != p->D) return DSV4_ERR_SHAPE;
  if (!(p->scale == p->scale)) return DSV4_ERR_ARG;
  if ((p->rope_q != 0 && p->rope_q != 1) || (p->rotate_out != 0 && p->rotate_out != 1)) return DSV4_ERR_ARG;
  return check_rope(p);
}

size_t scores_bytes(const dsv4_params* p) {
  const int64_t rows = (int64_t)p->B * p->Sq;
  if (rows == 0 || p->P_cap == 0 || p->nI < 1 || p->topk < 1) return 0;  // no indexer
  int64_t r = indexer_rows_per_chunk(rows, p->P_cap, kScoresBudget);
  if (r < 1) r = 1;
  size_t bytes = (size_t)r * p->P_cap * sizeof(float);
  // one query per sequence (decode): the fused scores + top-k kernel keeps each split's
  // candidates in the same space
  IndexerArgs a{};
  a.B = p->B; a.Sq = p->Sq; a.nI = p->nI; a.cI = p->cI; a.m = p->m; a.P_cap = p->P_cap; a.topk = p->topk;
  a.q_index = reinterpret_cast<const int32_t*>(16);  // decode plans use cache indices; never read
  if (p->Sq == 1 && indexer_tc_supported(a, p->dtype)) {
    const size_t sel = indexer_tc_select_bytes(a, r);
    if (sel > bytes) bytes = sel;
  }
  return bytes;
}

// idx kept in the workspace by dsv4_csa_layer (a prefill call: Sq == S).
size_t layer_idx_bytes(const dsv4_params* p) {
  if (p->Sq != p->S || p->nI < 1 || p->topk < 1) return 0;
  return (size_t)p->B * p->S * p->topk * sizeof(int32_t);
}

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

dsv4_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return DSV4_OK;
  if (e == cudaErrorNotSupported) return DSV4_ERR_SHAPE;
  return DSV4_ERR_CUDA;
}

dsv4_status run_compress(const dsv4_params* p, int c, const void* x, const void* z, const float* bias,
                         const int64_t* pos, int apply_rope, void* pool, void* x_rot, void* stream) {
  if (c < 2 || (c & 1)) return DSV4_ERR_SHAPE;
  const bool rotate_only = pool == nullptr && p->P_cap == 0;  // sliding-window layer: no pool
  if (!rotate_only && p->S / p->m > p->P_cap) return DSV4_ERR_SHAPE;
  if (!x || (!pool && !rotate_only) || (rotate_only && !x_rot)) return DSV4_ERR_ARG;
  if (!ok_ptr(x) || (pool && !aligned16(pool))) return DSV4_ERR_ALIGN;
  if ((z && !aligned16(z)) || (bias && !aligned16(bias)) || (x_rot && !aligned16(x_rot))) return DSV4_ERR_ALIGN;
  if (apply_rope != 0 && apply_rope != 1) return DSV4_ERR_ARG;
  if (apply_rope) {
    if (p->R < 0 || (p->R & 1) || p->R > c || p->R > 2 * kMaxRopePairs || !(p->rope_theta > 0.f))
      return DSV4_ERR_SHAPE;
    if (!pos) return DSV4_ERR_ARG;
    if (!aligned16(pos)) return DSV4_ERR_ALIGN;
  } else if (x_rot) {
    return DSV4_ERR_ARG;  // the rotated copy only exists with RoPE
  }
  CompressArgs a{};
  a.B = p->B; a.S = p->S; a.c = c; a.m = p->m; a.overlap = p->overlap; a.P_cap = p->P_cap;
  a.R = apply_rope ? p->R : 0; a.apply_rope = apply_rope; a.theta = p->rope_theta;
  a.x = x; a.z = z; a.bias = bias; a.pos = pos; a.pool = pool; a.x_rot = x_rot;
  return from_cuda(launch_compress(a, p->dtype, as_stream(stream)));
}

dsv4_status run_indexer(const dsv4_params* p, const void* qI, const float* wI, const void* poolI,
                        const int32_t* q_index, int32_t* idx, void* scores, size_t scores_cap, void* stream) {
  IndexerArgs a{};
  a.B = p->B; a.Sq = p->Sq; a.nI = p->nI; a.cI = p->cI; a.m = p->m; a.P_cap = p->P_cap; a.topk = p->topk;
  a.qI = qI; a.wI = wI; a.poolI = poolI; a.q_index = q_index; a.idx = idx;
  a.scores = static_cast<float*>(scores);
  a.scores_cap = scores_cap;
  const int64_t rows = (int64_t)p->B * p->Sq;
  a.rows_per_chunk = indexer_rows_per_chunk(rows, p->P_cap, scores_cap < kScoresBudget ? scores_cap : kScoresBudget);
  if (rows == 0) return DSV4_OK;
  if (a.rows_per_chunk < 1) return DSV4_ERR_WORKSPACE;
  return from_cuda(launch_indexer_topk(a, p->dtype, as_stream(stream)));
}

// Attention with given index lists (idx), every visible entry (idx and scores NULL), or lists
// the tensor-core kernel selects from score rows (scores, written to idx_out; the caller has
// checked attn_tc_selects).
dsv4_status run_attn(const dsv4_params* p, const void* q, const void* kv_win, const void* pool,
                     const int32_t* idx, const float* sink, const int64_t* qpos, const int32_t* q_index,
                     void* out, void* workspace, size_t ws_bytes, void* stream, const float* scores = nullptr,
                     int32_t* idx_out = nullptr) {
  AttnArgs a{};
  a.B = p->B; a.Sq = p->Sq; a.H = p->H; a.D = p->D; a.R = p->R; a.dv = p->dv; a.n_win = p->n_win;
  a.win_ring = p->win_ring; a.m = p->m; a.P_cap = p->P_cap; a.topk = p->topk; a.rope_q = p->rope_q;
  a.rotate_out = p->rotate_out; a.kv_rows = p->S; a.scale = p->scale; a.theta = p->rope_theta;
  a.q = q; a.kv_win = kv_win; a.pool = pool; a.idx = idx; a.sink = sink; a.qpos = qpos; a.q_index = q_index;
  a.out = out;
  a.part = nullptr;
  a.nsplit = 1;
  a.scores = scores;
  a.idx_out = idx_out;
  const int64_t rows = (int64_t)p->B * p->Sq;
  if (rows == 0) return DSV4_OK;
  if (idx && index_checks_on()) {
    const cudaError_t e = launch_index_check(idx, q_index, rows, p->Sq, p->topk, p->m, p->P_cap, as_stream(stream));
    if (e != cudaSuccess) return from_cuda(e);
  }
  if (scores && !attn_tc_selects(a, p->dtype)) return DSV4_ERR_SHAPE;
  if (attn_tc_supported(a, p->dtype)) {
    // few queries: split each query's keys over several CTAs when a workspace is given
    const size_t need = attn_split_bytes(rows, attn_keys_estimate(p), p->dv);
    if (need > 0 && workspace && ws_bytes >= need) {
      a.part = static_cast<float*>(workspace);
      a.nsplit = attn_splits(rows, attn_keys_estimate(p));
    }
    return from_cuda(launch_attn_tc(a, as_stream(stream)));
  }
  return from_cuda(launch_attn_simt(a, p->dtype, as_stream(stream)));
}

// The tensor-core attention can select each query's index list from its score row itself.
bool attn_selects(const dsv4_params* p, const void* pool) {
  AttnArgs a{};
  a.B = p->B; a.Sq = p->Sq; a.H = p->H; a.D = p->D; a.R = p->R; a.dv = p->dv; a.n_win = p->n_win;
  a.win_ring = p->win_ring; a.m = p->m; a.P_cap = p->P_cap; a.topk = p->topk; a.pool = pool;
  return attn_tc_selects(a, p->dtype);
}

dsv4_status check_attn_ptrs(const dsv4_params* p, const void* q, const void* kv_win, const void* pool,
                            const int32_t* idx, const float* sink, const int64_t* qpos, const int32_t* q_index,
                            const void* out) {
  if (!q || !sink || !out) return DSV4_ERR_ARG;
  if (p->n_win > 0 && !kv_win) return DSV4_ERR_ARG;
  if (!pool && (idx || p->P_cap > 0)) return DSV4_ERR_ARG;
  if ((p->rope_q || p->rotate_out) && !qpos) return DSV4_ERR_ARG;
  if (idx && p->topk < 1) return DSV4_ERR_SHAPE;
  if (!q_index && p->Sq > p->S && p->n_win > 0 && p->win_ring == 0) return DSV4_ERR_SHAPE;
  const void* ptrs[] = {q, kv_win, pool, idx, sink, qpos, q_index, out};
  for (const void* x : ptrs)
    if (x && !aligned16(x)) return DSV4_ERR_ALIGN;
  return DSV4_OK;
}

}  // namespace

extern "C" {

const char* dsv4_status_string(dsv4_status s) {
  switch (s) {
    case DSV4_OK: return "ok";
    case DSV4_ERR_ARG: return "invalid argument (null pointer or bad flag)";
    case DSV4_ERR_SHAPE: return "unsupported or inconsistent sizes";
    case DSV4_ERR_ALIGN: return "tensor pointer not 16-byte aligned";
    case DSV4_ERR_DTYPE: return "unknown dtype";
    case DSV4_ERR_CUDA: return "CUDA runtime error";
    case DSV4_ERR_DEVICE_CHECK: return "device-side check failed";
    case DSV4_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

int32_t dsv4_version(void) { return 100; }

uint64_t dsv4_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

dsv4_status dsv4_device_check(void* stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return DSV4_ERR_CUDA;
  int code = 0, code2 = 0, code3 = 0, code4 = 0;
  if (take_attn_tc_error(&code) != cudaSuccess) return DSV4_ERR_CUDA;
  if (take_indexer_tc_error(&code2) != cudaSuccess) return DSV4_ERR_CUDA;
  if (take_out_proj_error(&code3) != cudaSuccess) return DSV4_ERR_CUDA;
  if (take_index_check_error(&code4) != cudaSuccess) return DSV4_ERR_CUDA;
  return (code || code2 || code3 || code4) ? DSV4_ERR_DEVICE_CHECK : DSV4_OK;
}

void dsv4_set_index_checks(int32_t on) { set_index_checks(on); }

int32_t dsv4_index_checks(void) { return index_checks_on() ? 1 : 0;
}

size_t dsv4_workspace_bytes(const dsv4_params* p) {
  if (!p || check_common(p) != DSV4_OK) return 0;
  const size_t layer = align_up(layer_idx_bytes(p)) + align_up(scores_bytes(p));
  const size_t attn = align_up(attn_split_bytes((int64_t)p->B * p->Sq, attn_keys_estimate(p), p->dv));
  return layer > attn ? layer : attn;  // the attention partials reuse the indexer's scores space
}

dsv4_status dsv4_compress_kv(const dsv4_params* p, int32_t c, const void* x, const void* z, const float* bias,
                             const int64_t* pos, int32_t apply_rope, void* pool, void* x_rot, void* stream) {
  dsv4_status st = check_common(p);
  if (st != DSV4_OK) return st;
  return run_compress(p, c, x, z, bias, pos, apply_rope, pool, x_rot, stream);
}

dsv4_status dsv4_decode_append(const dsv4_params* p, int32_t c, const void* x, const void* z, const float* bias,
                               const int64_t* pos, const int32_t* t, void* buf_x, void* buf_z, int64_t* buf_pos,
                               int32_t apply_rope, void* win, void* pool, void* stream) {
  dsv4_status st = check_common(p);
  if (st != DSV4_OK) return st;
  if (c < 2 || (c & 1)) return DSV4_ERR_SHAPE;
  if (!x || !pos || !t || !buf_x || !buf_pos || !pool) return DSV4_ERR_ARG;
  if (z && !buf_z) return DSV4_ERR_ARG;  // logits can only be pooled from the buffer
  if (win && p->win_ring < 1) return DSV4_ERR_SHAPE;
  if (apply_rope != 0 && apply_rope != 1) return DSV4_ERR_ARG;
  if (apply_rope && (p->R < 0 || (p->R & 1) || p->R > c || p->R > 2 * kMaxRopePairs || !(p->rope_theta > 0.f)))
    return DSV4_ERR_SHAPE;
  const void* ptrs[] = {x, z, bias, pos, t, buf_x, buf_z, buf_pos, win, pool};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return DSV4_ERR_ALIGN;
  DecodeAppendArgs a{};
  a.B = p->B; a.c = c; a.m = p->m; a.overlap = p->overlap; a.win_ring = p->win_ring; a.P_cap = p->P_cap;
  a.R = apply_rope ? p->R : 0; a.apply_rope = apply_rope; a.theta = p->rope_theta;
  a.x = x; a.z = z; a.bias = bias; a.pos = pos; a.t = t; a.buf_x = buf_x; a.buf_z = buf_z; a.buf_pos = buf_pos;
  a.win = win; a.pool = pool;
  return from_cuda(launch_decode_append(a, p->dtype, as_stream(stream)));
}

dsv4_status dsv4_indexer_topk(const dsv4_params* p, const void* qI, const float* wI, const void* poolI,
                              const int32_t* q_index, int32_t* idx, void* workspace, size_t ws_bytes,
                              void* stream) {
  dsv4_status st = check_common(p);
  if (st != DSV4_OK) return st;
  if ((st = check_indexer(p)) != DSV4_OK) return st;
  if (!qI || !wI || !poolI || !idx) return DSV4_ERR_ARG;
  const void* ptrs[] = {qI, wI, poolI, q_index, idx, workspace};
  for (const void* x : ptrs)
    if (x && !aligned16(x)) return DSV4_ERR_ALIGN;
  if (!q_index && p->Sq > p->S) return DSV4_ERR_SHAPE;
  const size_t need = scores_bytes(p);
  if (need > 0 && (!workspace || ws_bytes < need)) return DSV4_ERR_WORKSPACE;
  return run_indexer(p, qI, wI, poolI, q_index, idx, workspace, ws_bytes, stream);
}

dsv4_status dsv4_indexer_topk_noalloc(const dsv4_params* p, const void* qI, const float* wI, const void* poolI,
                                      const int32_t* q_index, int32_t* idx, void* stream) {
  dsv4_status st = check_common(p);
  if (st != DSV4_OK) return st;
  if ((st = check_indexer(p)) != DSV4_OK) return st;
  if (!qI || !wI || !poolI || !idx) return DSV4_ERR_ARG;
  const void* ptrs[] = {qI, wI, poolI, q_index, idx};
  for (const void* x : ptrs)
    if (x && !aligned16(x)) return DSV4_ERR_ALIGN;
  if (!q_index && p->Sq > p->S) return DSV4_ERR_SHAPE;
  if ((int64_t)p->P_cap > kNoAllocScoreFloats) return DSV4_ERR_SHAPE;  // one score row must fit
  if ((int64_t)p->B * p->Sq == 0) return DSV4_OK;
  float* scratch = nullptr;
  if (noalloc_scores_scratch(&scratch) != cudaSuccess) return DSV4_ERR_CUDA;
  return run_indexer(p, qI, wI, poolI, q_index, idx, scratch, (size_t)kNoAllocScoreFloats * sizeof(float), stream);
}

// Rows of one launch of the split entry points (the score grids' y extents stay below 65536).
dsv4_status dsv4_indexer_scores(const dsv4_params* p, const void* qI, const float* wI, const void* poolI,
                                const int32_t* q_index, float* scores, void* stream) {
  dsv4_status st = check_common(p);
  if (st != DSV4_OK) return st;
  if ((st = check_indexer(p)) != DSV4_OK) return st;
  if (!qI || !wI || !poolI || !scores) return DSV4_ERR_ARG;
  const void* ptrs[] = {qI, wI, poolI, q_index, scores};
  for (const void* x : ptrs)
    if (x && !aligned16(x)) return DSV4_ERR_ALIGN;
  if (!q_index && p->Sq > p->S) return DSV4_ERR_SHAPE;
  IndexerArgs a{};
  a.B = p->B; a.Sq = p->Sq; a.nI = p->nI; a.cI = p->cI; a.m = p->m; a.P_cap = p->P_cap; a.topk = p->topk;
  a.qI = qI; a.wI = wI; a.poolI = poolI; a.q_index = q_index;
  const int64_t rows = (int64_t)p->B * p->Sq;
  for (int64_t r0 = 0; r0 < rows; r0 += kSplitChunkRows) {
    const int64_t r1 = r0 + kSplitChunkRows < rows ? r0 + kSplitChunkRows : rows;
    a.scores = scores + r0 * (int64_t)p->P_cap;
    a.rows_per_chunk = r1 - r0;
    const cudaError_t e = launch_indexer_scores(a, p->dtype, r0, r1, as_stream(stream));
    if (e != cudaSuccess) return from_cuda(e);
  }
  return DSV4_OK;
}

dsv4_status dsv4_topk_select(const dsv4_params* p, const float* scores, const int32_t* q_index, int32_t* idx,
                             void* stream) {
  dsv4_status st = check_common(p);
  if (st != DSV4_OK) return st;
  if (p->topk < 1 || p->P_cap < 1) return DSV4_ERR_SHAPE;
  if (!scores || !idx) return DSV4_ERR_ARG;
  const void* ptrs[] = {scores, q_index, idx};
  for (const void* x : ptrs)
    if (x && !aligned16(x)) return DSV4_ERR_ALIGN;
  if (!q_index && p->Sq > p->S) return DSV4_ERR_SHAPE;
  IndexerArgs a{};
  a.B = p->B; a.Sq = p->Sq; a.nI = p->nI; a.cI = p->cI; a.m = p->m; a.P_cap = p->P_cap; a.topk = p->topk;
  a.q_index = q_index; a.idx = idx;
  const int64_t rows = (int64_t)p->B * p->Sq;
  for (int64_t r0 = 0; r0 < rows; r0 += kSplitChunkRows) {
    const int64_t r1 = r0 + kSplitChunkRows < rows ? r0 + kSplitChunkRows : rows;
    a.scores = const_cast<float*>(scores) + r0 * (int64_t)p->P_cap;
    a.rows_per_chunk = r1 - r0;
    const cudaError_t e = launch_topk(a, r0, r1, as_stream(stream));
    if (e != cudaSuccess) return from_cuda(e);
  }
  return DSV4_OK;
}

dsv4_status dsv4_sparse_mqa_attn(const dsv4_params* p, const void* q, const void* kv_win, const void* pool,
                                 const int32_t* idx, const float* sink, const int64_t* qpos,
                                 const int32_t* q_index, void* out, void* workspace, size_t ws_bytes,
                                 void* stream) {
  dsv4_status st = check_common(p);
  if (st != DSV4_OK) return st;
  if ((st = check_attn(p)) != DSV4_OK) return st;
  if ((st = check_attn_ptrs(p, q, kv_win, pool, idx, sink, qpos, q_index, out)) != DSV4_OK) return st;
  return run_attn(p, q, kv_win, pool, idx, sink, qpos, q_index, out, workspace, ws_bytes, stream);
}

dsv4_status dsv4_sparse_mqa_attn_scores(const dsv4_params* p, const void* q, const void* kv_win, const void* pool,
                                        const float* scores, const float* sink, const int64_t* qpos,
                                        const int32_t* q_index, int32_t* idx, void* out, void* workspace,
                                        size_t ws_bytes, void* stream) {
  dsv4_status st = check_common(p);
  if (st != DSV4_OK) return st;
  if ((st = check_attn(p)) != DSV4_OK) return st;
  if (!scores || !idx) return DSV4_ERR_ARG;
  if (p->topk < 1 || p->P_cap < 1) return DSV4_ERR_SHAPE;
  if ((st = check_attn_ptrs(p, q, kv_win, pool, idx, sink, qpos, q_index, out)) != DSV4_OK) return st;
  if (!aligned16(scores)) return DSV4_ERR_ALIGN;
  if (!q_index && p->Sq > p->S) return DSV4_ERR_SHAPE;
  if (attn_selects(p, pool))
    return run_attn(p, q, kv_win, pool, nullptr, sink, qpos, q_index, out, workspace, ws_bytes, stream, scores, idx);
  // otherwise the two calls this one stands for
  if ((st = dsv4_topk_select(p, scores, q_index, idx, stream)) != DSV4_OK) return st;
  return run_attn(p, q, kv_win, pool, idx, sink, qpos, q_index, out, workspace, ws_bytes, stream);
}

dsv4_status dsv4_csa_layer(const dsv4_params* p, const void* q, const void* kv, const void* z, const float* bias,
                           const void* qI, const float* wI, const void* kI, const void* zI, const float* biasI,
                           const float* sink, const int64_t* pos, void* out, void* pool, void* poolI,
                           void* kv_rot, int32_t* idx, void* workspace, size_t ws_bytes, void* stream) {
  dsv4_status st = check_common(p);
  if (st != DSV4_OK) return st;
  if (p->Sq != p->S || p->win_ring != 0 || p->rope_q != 1) return DSV4_ERR_SHAPE;
  if ((st = check_attn(p)) != DSV4_OK) return st;
  if ((st = check_indexer(p)) != DSV4_OK) return st;
  if (!q || !kv || !qI || !wI || !kI || !sink || !pos || !out || !pool || !poolI || !kv_rot) return DSV4_ERR_ARG;
  const void* ptrs[] = {q, kv, z, bias, qI, wI, kI, zI, biasI, sink, pos, out, pool, poolI, kv_rot, idx, workspace};
  for (const void* x : ptrs)
    if (x && !aligned16(x)) return DSV4_ERR_ALIGN;
  if (p->S / p->m > p->P_cap) return DSV4_ERR_SHAPE;
  const size_t need = dsv4_workspace_bytes(p);
  if (need > 0 && (!workspace || ws_bytes < need)) return DSV4_ERR_WORKSPACE;
  char* ws = static_cast<char*>(workspace);
  int32_t* idx_buf = idx ? idx : reinterpret_cast<int32_t*>(ws);
  char* scores = ws + align_up(layer_idx_bytes(p));
  const size_t scores_cap = ws_bytes - align_up(layer_idx_bytes(p));

  if ((st = run_compress(p, p->D, kv, z, bias, pos, 1, pool, kv_rot, stream)) != DSV4_OK) return st;
  if ((st = run_compress(p, p->cI, kI, zI, biasI, pos, 0, poolI, nullptr, stream)) != DSV4_OK) return st;
  const int64_t rows = (int64_t)p->B * p->Sq;
  if (attn_selects(p, pool) && scores_cap / sizeof(float) / (size_t)p->P_cap >= (size_t)rows &&
      rows <= kSplitChunkRows) {
    // every score row at once, then the attention selects each query's list itself
    IndexerArgs ia{};
    ia.B = p->B; ia.Sq = p->Sq; ia.nI = p->nI; ia.cI = p->cI; ia.m = p->m; ia.P_cap = p->P_cap; ia.topk = p->topk;
    ia.qI = qI; ia.wI = wI; ia.poolI = poolI; ia.scores = reinterpret_cast<float*>(scores); ia.rows_per_chunk = rows;
    const cudaError_t e = launch_indexer_scores(ia, p->dtype, 0, rows, as_stream(stream));
    if (e != cudaSuccess) return from_cuda(e);
    return run_attn(p, q, kv_rot, pool, nullptr, sink, pos, nullptr, out, nullptr, 0, stream,
                    reinterpret_cast<const float*>(scores), idx_buf);
  }
  if ((st = run_indexer(p, qI, wI, poolI, nullptr, idx_buf, scores, scores_cap, stream)) != DSV4_OK) return st;
  return run_attn(p, q, kv_rot, pool, idx_buf, sink, pos, nullptr, out, nullptr, 0, stream);
}

dsv4_status dsv4_hca_layer(const dsv4_params* p, const void* q, const void* kv, const void* z, const float* bias,
                           const float* sink, const int64_t* pos, void* out, void* pool, void* kv_rot,
                           void* workspace, size_t ws_bytes, void* stream) {
  (void)workspace;
  (void)ws_bytes;
  dsv4_status st = check_common(p);
  if (st != DSV4_OK) return st;
  if (p->Sq != p->S || p->win_ring != 0 || p->rope_q != 1 || p->overlap != 0) return DSV4_ERR_SHAPE;
  if ((st = check_attn(p)) != DSV4_OK) return st;
  if (!q || !kv || !sink || !pos || !out || !pool || !kv_rot) return DSV4_ERR_ARG;
  const void* ptrs[] = {q, kv, z, bias, sink, pos, out, pool, kv_rot};
  for (const void* x : ptrs)
    if (x && !aligned16(x)) return DSV4_ERR_ALIGN;
  if (p->S / p->m > p->P_cap) return DSV4_ERR_SHAPE;
  if ((st = run_compress(p, p->D, kv, z, bias, pos, 1, pool, kv_rot, stream)) != DSV4_OK) return st;
  return run_attn(p, q, kv_rot, pool, nullptr, sink, pos, nullptr, out, nullptr, 0, stream);
}

dsv4_status dsv4_grouped_out_proj(const dsv4_params* p, int32_t T, int32_t groups, int32_t dg, int32_t hidden,
                                  const void* o, const void* wa, const void* wb, void* u, void* y, void* stream) {
  if (!p) return DSV4_ERR_ARG;
  if (p->dtype != DSV4_BF16) return p->dtype == DSV4_F32 ? DSV4_ERR_SHAPE : DSV4_ERR_DTYPE;
  if (T < 0 || groups < 1 || dg < 1 || hidden < 1 || p->H < 1 || p->dv < 1) return DSV4_ERR_SHAPE;
  if (p->H % groups != 0) return DSV4_ERR_SHAPE;
  if (!o || !wa || !wb || !u || !y) return DSV4_ERR_ARG;
  const void* ptrs[] = {o, wa, wb, u, y};
  for (const void* x : ptrs)
    if (!aligned16(x)) return DSV4_ERR_ALIGN;
  OutProjArgs a{};
  a.T = T; a.H = p->H; a.dv = p->dv; a.groups = groups; a.dg = dg; a.hidden = hidden;
  a.o = o; a.wa = wa; a.wb = wb; a.u = u; a.y = y;
  if (!out_proj_supported(a)) return DSV4_ERR_SHAPE;
  return from_cuda(launch_out_proj(a, as_stream(stream)));
}

}  // extern "C"
