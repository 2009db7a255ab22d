// Launchers shared between the C-ABI layer (dsv4_api.cu) and the kernel files.
// Arguments arrive validated; each launcher returns the cudaGetLastError() of its launches.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "dsv4.h"

namespace dsv4 {

// Count one kernel launch (read back by dsv4_launch_count).
void note_launch(int n = 1);

// RoPE frequencies theta^(-2k/R), k < R/2, formed on the host in double precision (R <= 128).
constexpr int kMaxRopePairs = 64;

struct CompressArgs {
  int B, S, c, m, overlap, P_cap, R, apply_rope;
  float theta;
  double inv_freq[kMaxRopePairs];  // filled by the launcher
  const void* x;
  const void* z;
  const float* bias;
  const int64_t* pos;
  void* pool;
  void* x_rot;
};
cudaError_t launch_compress(const CompressArgs& a, int dtype, cudaStream_t st);

struct DecodeAppendArgs {
  int B, c, m, overlap, win_ring, P_cap, R, apply_rope;
  float theta;
  double inv_freq[kMaxRopePairs];  // filled by the launcher
  const void* x;
  const void* z;
  const float* bias;
  const int64_t* pos;
  const int32_t* t;
  void* buf_x;
  void* buf_z;
  int64_t* buf_pos;
  void* win;
  void* pool;
};
cudaError_t launch_decode_append(const DecodeAppendArgs& a, int dtype, cudaStream_t st);

struct IndexerArgs {
  int B, Sq, nI, cI, m, P_cap, topk;
  const void* qI;
  const float* wI;
  const void* poolI;
  const int32_t* q_index;
  int32_t* idx;
  float* scores;        // workspace: [rows_per_chunk, P_cap] fp32
  int64_t rows_per_chunk;
  size_t scores_cap;    // bytes at `scores` (the fused decode path keeps its candidates there)
};
cudaError_t launch_indexer_topk(const IndexerArgs& a, int dtype, cudaStream_t st);
// The two halves of launch_indexer_topk for query rows [r0, r1): score row r lives at
// a.scores + (r - r0) * P_cap (entries w < vis written, the rest untouched).
cudaError_t launch_indexer_scores(const IndexerArgs& a, int dtype, int64_t r0, int64_t r1, cudaStream_t st);
cudaError_t launch_topk(const IndexerArgs& a, int64_t r0, int64_t r1, cudaStream_t st);
// Tensor-core score kernel (bf16): scores of rows [r0, r1) into a.scores.
bool indexer_tc_supported(const IndexerArgs& a, int dtype);
cudaError_t launch_indexer_tc_scores(const IndexerArgs& a, int64_t r0, int64_t r1, cudaStream_t st);
// Fused scores + top-k for one query per sequence (decode); a.scores is ws_bytes of work space.
// cudaErrorNotSupported when the shapes or the work space do not allow it.
cudaError_t launch_indexer_tc_select(const IndexerArgs& a, int64_t r0, int64_t r1, size_t ws_bytes,
                                     cudaStream_t st);
// Work space the fused path needs for `rows` queries of one query per sequence (0: the path
// does not apply to these shapes).
size_t indexer_tc_select_bytes(const IndexerArgs& a, int64_t rows);
cudaError_t take_indexer_tc_error(int* code);
// Rows of queries whose scores fit in `bytes` of score workspace.
int64_t indexer_rows_per_chunk(int64_t total_rows, int P_cap, size_t bytes);
// Device address (on the current device) of the fixed score scratch used by
// dsv4_indexer_topk_noalloc; set up on the first call per device.
constexpr int64_t kNoAllocScoreFloats = int64_t(4) << 20;  // 16 MiB of fp32 scores
cudaError_t noalloc_scores_scratch(float** ptr);

struct AttnArgs {
  int B, Sq, H, D, R, dv, n_win, win_ring, m, P_cap, topk, rope_q, rotate_out, kv_rows;
  float scale, theta;
  const void* q;
  const void* kv_win;
  const void* pool;
  const int32_t* idx;
  const float* sink;
  const int64_t* qpos;
  const int32_t* q_index;
  void* out;
  float* part;  // split-over-keys partials (workspace) or nullptr
  int nsplit;   // key splits per query (1 = no split)
  // Score rows [B*Sq, P_cap] f32 (idx then NULL): each query's index list is selected from its
  // row inside the attention kernel, as dsv4_topk_select would, and written to idx_out.
  const float* scores;
  int32_t* idx_out;
};
// Key splits per query used by the tensor-core attention for B*Sq queries attending about
// keys_per_query keys each (a pure function of the sizes, so that the workspace size is one
// too), and the workspace it needs.
int attn_splits(int64_t rows, int64_t keys_per_query);
size_t attn_split_bytes(int64_t rows, int64_t keys_per_query, int dv);
cudaError_t launch_attn_simt(const AttnArgs& a, int dtype, cudaStream_t st);
// Tensor-core (tcgen05) path; returns cudaErrorNotSupported when the shape is not covered.
bool attn_tc_supported(const AttnArgs& a, int dtype);
// The tensor-core kernel can select the index lists from score rows (a.scores) itself.
bool attn_tc_selects(const AttnArgs& a, int dtype);
cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t st);
// Read and clear the tensor-core kernel's error word (non-zero: a bounded wait gave up).
cudaError_t take_attn_tc_error(int* code);

// Grouped output projection (bf16, tensor cores): u = per-group o_a_proj of the attention
// output, y = o_b_proj(u).
struct OutProjArgs {
  int T, H, dv, groups, dg, hidden;
  const void* o;   // [T, H, dv]
  const void* wa;  // [groups, dg, (H/groups)*dv]
  const void* wb;  // [hidden, groups*dg]
  void* u;         // [T, groups*dg]
  void* y;         // [T, hidden]
};
bool out_proj_supported(const OutProjArgs& a);
cudaError_t launch_out_proj(const OutProjArgs& a, cudaStream_t st);
cudaError_t take_out_proj_error(int* code);

// Optional validation of attention index lists (out of range, not visible, duplicated):
// off by default (on in DSV4_DEBUG builds), switched by dsv4_set_index_checks.
void set_index_checks(int on);
bool index_checks_on();
cudaError_t launch_index_check(const int32_t* idx, const int32_t* q_index, int64_t rows, int Sq, int topk, int m,
                               int P_cap, cudaStream_t st);
cudaError_t take_index_check_error(int* code);

}  // namespace dsv4
