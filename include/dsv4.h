/*
 * dsv4.h — C ABI of libdsv4, the DeepSeek-V4 hybrid compressed attention core
 * (CSA / HCA, and the token-level DSA variant) on NVIDIA B200 (sm_100a).
 *
 * Method sources (HF Transformers model docs):
 *   [V4]  "DeepSeek-V4" doc: section "Architecture (paper §2)" → "Hybrid attention
 *         (§2.3)" (CSA / HCA items, shared K=V MQA, partial RoPE and the -i output
 *         rotation of eq. 26, per-head sink of eq. 27, sliding-window K=V branch),
 *         "Attention mask layout" (visibility rules, -1 sentinels), "Cache layers",
 *         and the DeepseekV4Config parameters (sliding_window, compress_rates,
 *         compress_rope_theta, index_n_heads, index_head_dim, index_topk).
 *   [V32] "DeepSeek-V3.2" doc: section "DeepSeek Sparse Attention (DSA)"
 *         (Lightning Indexer, fine-grained top-k token selection).
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; they must be
 *     16-byte aligned and the tensors contiguous, row-major, in the shapes given.
 *     "T" is the activation dtype named by params->dtype (float32 or bfloat16).
 *   - The library allocates no memory and keeps no state between calls.  Scratch
 *     space is the caller's `workspace` of at least dsv4_workspace_bytes(params).
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  Arguments are validated on the host before any launch;
 *     an invalid call returns a non-zero dsv4_status and enqueues nothing.
 *   - No entry point aborts, traps or synchronises the device.  DSV4_ERR_CUDA
 *     means a launch was refused by the runtime (cudaGetLastError).
 *
 * Index conventions
 *   - Cache index t of a query decides visibility; RoPE positions (pos, qpos)
 *     only feed the rotations, so shifting every position leaves outputs unchanged.
 *   - A query at cache index t sees pool entries w < min((t+1)/m, P_cap) ([V4]
 *     "Attention mask layout": an entry is visible once its window has closed) and
 *     the window tokens (t - n_win, t] ∩ [0, t].
 */
#ifndef DSV4_H_
#define DSV4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSV4_OK = 0,
  DSV4_ERR_ARG = 1,          /* null pointer where one is required, or bad flag value */
  DSV4_ERR_SHAPE = 2,        /* sizes inconsistent or outside what the kernels support */
  DSV4_ERR_ALIGN = 3,        /* a tensor pointer is not 16-byte aligned */
  DSV4_ERR_DTYPE = 4,        /* unknown params->dtype */
  DSV4_ERR_CUDA = 5,         /* the CUDA runtime refused a launch or query */
  DSV4_ERR_DEVICE_CHECK = 6, /* dsv4_device_check: a kernel gave up a bounded wait */
  DSV4_ERR_WORKSPACE = 7     /* workspace missing or smaller than dsv4_workspace_bytes() */
} dsv4_status;

typedef enum { DSV4_F32 = 0, DSV4_BF16 = 1 } dsv4_dtype;

/* Sizes of one call.  Nothing has a hidden default: the caller sets every field. */
typedef struct dsv4_params {
  int32_t B;          /* sequences in the batch */
  int32_t S;          /* tokens per sequence in kv / kI / x (prefill and compress) */
  int32_t Sq;         /* query tokens per sequence */
  int32_t H;          /* query heads (num_attention_heads); one shared K=V head */
  int32_t D;          /* head_dim: width of q rows and K=V rows */
  int32_t R;          /* trailing rotary channels (qk_rope_head_dim), even, <= D */
  int32_t dv;         /* value width: the first dv channels of each K=V row */
  int32_t n_win;      /* sliding_window (0 = no window branch) */
  int32_t win_ring;   /* 0: window rows addressed by cache index in [B,S,D];
                         >0: ring buffer [B,win_ring,D], token j in slot j % win_ring
                         (requires win_ring >= n_win) */
  int32_t m;          /* compression rate (compress_rates: 4 CSA, 128 HCA, 1 DSA) */
  int32_t overlap;    /* 1: entry w pools tokens [(w-1)m,(w+1)m) (CSA); 0: [wm,(w+1)m) */
  int32_t P_cap;      /* pool capacity: entries per sequence in pool / poolI buffers */
  int32_t nI;         /* index_n_heads */
  int32_t cI;         /* index_head_dim */
  int32_t topk;       /* index_topk */
  float scale;        /* softmax scale applied to q.k (e.g. 1/sqrt(D)) */
  float rope_theta;   /* RoPE base (compress_rope_theta for CSA/HCA, rope_theta for DSA) */
  int32_t rope_q;     /* 1: rotate q at qpos inside the attention; 0: q already rotated */
  int32_t rotate_out; /* 1: rotate the output rope slice by -qpos (eq. 26); needs dv == D */
  int32_t dtype;      /* dsv4_dtype of every activation tensor "T" */
} dsv4_params;

/*
 * KV compressor ([V4] "Hybrid attention (§2.3)", CSA item: low-compression pool with
 * overlapping windows; HCA item: high-compression pool, non-overlapping windows;
 * "Cache layers": the indexer keys get their own pool at index_head_dim).
 *
 * Pools token rows x into entries: for each entry w < S/m and channel d,
 *   pool[w,d] = sum_{j in J_w} alpha_j[d] x[j,d],
 *   alpha_.[d] = softmax over J_w of (z[j,d] + bias[slot(j),d]),
 * with J_w = [(w-1)m, (w+1)m) ∩ [0,S) and slot(j) = j-(w-1)m when overlap, else
 * J_w = [wm,(w+1)m), slot(j) = j-wm.  With apply_rope, the entry's trailing R channels
 * are rotated (interleaved pairs, base rope_theta; R <= 128) at pos[b, w*m].
 *
 *   c      channels per row (D for the K=V stream, cI for the indexer-key stream)
 *   x      [B,S,c] T          token rows (not rotated)
 *   z      [B,S,c] T or NULL  per-token compressor logits (NULL = 0)
 *   bias   [2m or m, c] f32 or NULL   per-slot bias (NULL = 0)
 *   pos    [B,S] int64        RoPE positions (required when apply_rope)
 *   pool   [B,P_cap,c] T      out: entries 0 .. S/m-1 are written (S/m <= P_cap)
 *   x_rot  [B,S,c] T or NULL  out: x rotated at pos (the window keys); needs apply_rope
 * A sliding-window layer ([V4] layer types, `sliding_attention`) keeps no pool: with
 * P_cap == 0 and pool == NULL the call only writes x_rot (which is then required).
 */
dsv4_status dsv4_compress_kv(const dsv4_params* params, int32_t c, const void* x, const void* z,
                             const float* bias, const int64_t* pos, int32_t apply_rope,
                             void* pool, void* x_rot, void* stream);

/*
 * Decode-cache append ([V4] "Cache layers": the CSA / HCA cache keeps the sliding window of
 * K=V rows and the compressor's buffer of the tokens of the open window(s) -- for CSA the
 * previous block too, its overlap state; an entry is emitted every m tokens; the indexer
 * keys keep a buffer and a pool of their own).
 *
 * Appends one token to each of B sequences.  Sequence b's new token has cache index t[b]
 * (t[b] < 0: the sequence is skipped); the tokens of a sequence must be appended in order
 * t = 0, 1, 2, ...  When the token closes a block ((t+1) % m == 0), entry w = (t+1)/m - 1 is
 * pooled from the buffer and written if w < P_cap: the same pooling and RoPE as
 * dsv4_compress_kv, with the same arithmetic, so the entry has the same bits as the one
 * dsv4_compress_kv writes for the same token rows.  Lw = 2m with overlap, else m.
 *
 *   c          channels per row (D for the K=V stream, cI for the indexer keys); even
 *   x          [B,c] T             the new tokens' rows (not rotated)
 *   z          [B,c] T or NULL     their compressor logits (NULL = 0)
 *   bias       [Lw,c] f32 or NULL  per-slot bias
 *   pos        [B] int64           the new tokens' positions
 *   t          [B] int32           the new tokens' cache indices
 *   buf_x      [B,Lw,c] T          in/out: raw rows of the last Lw tokens (token j in slot j % Lw)
 *   buf_z      [B,Lw,c] T or NULL  in/out: their logits (required when z is given)
 *   buf_pos    [B,Lw] int64        in/out: their positions
 *   apply_rope rotate the window rows and the new entries (trailing R <= 128 channels, rope_theta)
 *   win        [B,win_ring,c] T or NULL  in/out: window ring; token j, rotated at its
 *                                  position when apply_rope, in slot j % win_ring
 *   pool       [B,P_cap,c] T       in/out: the pool
 * Uses B, m, overlap, win_ring, P_cap, R, rope_theta and dtype from params.  Validates on the
 * host (DSV4_ERR_ARG / _SHAPE / _ALIGN / _DTYPE) before any launch; allocates nothing.
 */
dsv4_status dsv4_decode_append(const dsv4_params* params, int32_t c, const void* x, const void* z,
                               const float* bias, const int64_t* pos, const int32_t* t, void* buf_x,
                               void* buf_z, int64_t* buf_pos, int32_t apply_rope, void* win, void* pool,
                               void* stream);

/*
 * Lightning Indexer + top-k ([V4] CSA item, eqs. 13-17 and index_topk (eq. 17);
 * [V32] DSA items 1-2).  For each query (b,s) at cache index t = q_index[b,s] and
 * every visible entry w < vis = min((t+1)/m, P_cap):
 *   I[w] = sum_h wI[b,s,h] * relu(qI[b,s,h,:] . poolI[b,w,:])
 * then keeps the min(topk, vis) entries of highest I (ties: lower w wins).
 *
 *   qI      [B,Sq,nI,cI] T
 *   wI      [B,Sq,nI] f32       per-head index weights
 *   poolI   [B,P_cap,cI] T      compressed indexer keys (no RoPE)
 *   q_index [B,Sq] int32 or NULL  cache index of each query (NULL: q_index[b,s] = s)
 *   idx     [B,Sq,topk] int32   out: selected entries in ASCENDING entry order, then -1
 *   workspace, ws_bytes         >= dsv4_workspace_bytes(params)
 * With one query per sequence (Sq == 1, bf16, nI <= 16), about a million scored entries
 * or more per call and a device that lets a CTA opt in to ~216 KB of shared memory (B200:
 * 227 KB), scores and selection run in one kernel whose score rows never leave shared
 * memory ([V32] DSA item 2); the index rows are the same, bit for bit.
 */
dsv4_status dsv4_indexer_topk(const dsv4_params* params, const void* qI, const float* wI,
                              const void* poolI, const int32_t* q_index, int32_t* idx,
                              void* workspace, size_t ws_bytes, void* stream);

/*
 * Allocation-free variant of dsv4_indexer_topk (the method has no counterpart: this is a
 * deployment convenience).  It is for callers that cannot hand the library a workspace:
 * plugin hosts that own all device memory and expose no allocator to the kernels they
 * call, and decode loops that must not call cudaMalloc / cudaFree because those calls can
 * synchronise the whole device.  Same arguments, results and ordering as
 * dsv4_indexer_topk, minus the workspace: the fp32 score rows live in a fixed 16 MiB
 * array of device memory inside the library (4,194,304 scores; every GPU that loads the
 * library holds it until the process exits), processed in chunks of whole query rows.
 *   - P_cap above 4,194,304 is rejected with DSV4_ERR_SHAPE (one score row must fit).
 *   - The first call on a device looks up that device's copy of the array
 *     (cudaGetSymbolAddress, with the device current); make that first call before any
 *     stream capture.  It allocates nothing, then or later.
 *   - Every call shares the array.  Calls that overlap on the GPU (other streams, other
 *     host threads) race on it and must be serialised by the caller.  No part of the
 *     array needs to start at zero: each score row is written before it is read.
 *   - The looked-up address is kept for the life of the process.  After cudaDeviceReset
 *     (or anything else that destroys and recreates the device's primary context) it is
 *     stale: do not call this entry point on that device again in the same process.
 */
dsv4_status dsv4_indexer_topk_noalloc(const dsv4_params* params, const void* qI, const float* wI,
                                      const void* poolI, const int32_t* q_index, int32_t* idx,
                                      void* stream);

/*
 * The two halves of dsv4_indexer_topk as separate calls, for callers that keep the score
 * rows (to inspect them, reuse them, or bring their own selection) and for timing each
 * kernel alone.  Same definitions as dsv4_indexer_topk ([V4] CSA item, Lightning Indexer
 * eqs. 13-17; [V32] DSA items 1-2).
 *
 * dsv4_indexer_scores: scores[b*Sq+s, w] = I[w] for every visible entry w < vis (vis as
 * above); entries w >= vis of a row are left untouched.
 *   qI, wI, poolI, q_index  as for dsv4_indexer_topk
 *   scores  [B*Sq, P_cap] f32, caller-owned, 16-byte aligned
 *
 * dsv4_topk_select: idx[b,s,:] = the min(topk, vis) entries w < vis with the highest
 * scores[b*Sq+s, w], in ascending entry order, then -1 (ties: lower w wins; -0 equals +0;
 * a NaN ranks above +inf when its sign bit is clear and below -inf when it is set).  Only
 * entries w < vis of each row are read.  Uses m, P_cap, topk, B, Sq (and S when q_index is
 * NULL) from params; nI and cI are not read.
 *   scores  [B*Sq, P_cap] f32
 *   idx     [B,Sq,topk] int32 out
 * Both validate on the host (DSV4_ERR_ARG / _SHAPE / _ALIGN) before any launch, allocate
 * nothing and are asynchronous on `stream`.
 */
dsv4_status dsv4_indexer_scores(const dsv4_params* params, const void* qI, const float* wI,
                                const void* poolI, const int32_t* q_index, float* scores,
                                void* stream);
dsv4_status dsv4_topk_select(const dsv4_params* params, const float* scores,
                             const int32_t* q_index, int32_t* idx, void* stream);

/*
 * Sparse shared-K=V MQA attention with sink ([V4] "Hybrid attention (§2.3)": one KV
 * head read as key and value, partial RoPE, -i output rotation (eq. 26), per-head sink
 * (eq. 27), sliding-window K=V branch concatenated with the compressor entries).
 * For query (b,s) at cache index t and head h, the keys are the window rows of tokens
 * (t-n_win, t] followed by the pool entries idx[b,s,:] that are >= 0; each key row k
 * is also its value v = k[0:dv]:
 *   l_j = scale * <q_h, k_j>,   o_h = sum_j e^{l_j} v_j / (e^{sink_h} + sum_j e^{l_j})
 *
 *   q       [B,Sq,H,D] T       rotated at qpos inside when rope_q (else already rotated)
 *   kv_win  window rows, already rotated: [B,S,D] T (win_ring == 0) or [B,win_ring,D] T
 *   pool    [B,P_cap,D] T      compressed entries, already rotated; NULL with P_cap == 0
 *                              and idx NULL: a sliding-window layer ([V4] layer types,
 *                              `sliding_attention`) attends the window alone
 *   idx     [B,Sq,topk] int32 or NULL   selected entries (-1 = empty slot); every entry
 *                              must be visible and appear once.  NULL: every visible
 *                              entry is attended (HCA, no indexer).
 *   sink    [H] f32            per-head sink logits
 *   qpos    [B,Sq] int64       RoPE position of each query (needed if rope_q/rotate_out)
 *   q_index [B,Sq] int32 or NULL   cache index of each query (NULL: s); with
 *                              win_ring == 0 window tokens at or past S select nothing
 *   out     [B,Sq,H,dv] T
 *   workspace, ws_bytes   optional: with fewer than 148 queries (decode) and a workspace of at
 *                              least dsv4_workspace_bytes(params), each query's keys are split
 *                              over several CTAs whose partial results are merged at the end
 */
dsv4_status dsv4_sparse_mqa_attn(const dsv4_params* params, const void* q, const void* kv_win,
                                 const void* pool, const int32_t* idx, const float* sink,
                                 const int64_t* qpos, const int32_t* q_index, void* out,
                                 void* workspace, size_t ws_bytes, void* stream);

/*
 * dsv4_topk_select followed by dsv4_sparse_mqa_attn, in one call ([V4] "Hybrid attention
 * (§2.3)", CSA item: the indexer's top index_topk entries of each query go straight into core
 * attention).  Same results as the two calls, bit for bit in idx:
 *   idx[b,s,:] = the min(topk, vis) entries w < vis with the highest scores[b*Sq+s, w], in
 *                ascending entry order, then -1 (ties: lower w wins; -0 equals +0),
 *   out        = dsv4_sparse_mqa_attn(params, q, kv_win, pool, idx, sink, qpos, q_index, ...).
 *   scores  [B*Sq, P_cap] f32   as written by dsv4_indexer_scores; entries w < vis are read
 *   idx     [B,Sq,topk] int32   out (caller-owned): the selected lists
 *   other arguments as for dsv4_sparse_mqa_attn (pool is required)
 * For bf16 with P_cap <= 2048 and topk <= 512 the attention kernel selects each query's list
 * from its score row itself (kept in shared memory; no selection launch, no list read back);
 * otherwise the call runs the two kernels.  Validates on the host (DSV4_ERR_ARG / _SHAPE /
 * _ALIGN) before any launch; asynchronous on `stream`.
 */
dsv4_status dsv4_sparse_mqa_attn_scores(const dsv4_params* params, const void* q, const void* kv_win,
                                        const void* pool, const float* scores, const float* sink,
                                        const int64_t* qpos, const int32_t* q_index, int32_t* idx,
                                        void* out, void* workspace, size_t ws_bytes, void* stream);

/*
 * One CSA layer in prefill (Sq == S, query s at cache index s, RoPE position pos[b,s]):
 * compress kv -> pool (rotated) and kv_rot (window keys), compress kI -> poolI,
 * indexer + top-k -> idx, sparse attention -> out.  With m == 1, overlap == 0,
 * n_win == 0 this is the token-level DSA layer of [V32].
 *   q [B,S,H,D] T (not rotated); kv [B,S,D] T; z [B,S,D] T or NULL; bias [Lw,D] f32 or NULL
 *   qI [B,S,nI,cI] T; wI [B,S,nI] f32; kI [B,S,cI] T; zI [B,S,cI] T or NULL;
 *   biasI [Lw,cI] f32 or NULL; sink [H] f32; pos [B,S] int64
 *   out [B,S,H,dv] T; pool [B,P_cap,D] T; poolI [B,P_cap,cI] T; kv_rot [B,S,D] T
 *   idx [B,S,topk] int32 or NULL (NULL: kept in the workspace)
 */
dsv4_status dsv4_csa_layer(const dsv4_params* params, const void* q, const void* kv,
                           const void* z, const float* bias, const void* qI, const float* wI,
                           const void* kI, const void* zI, const float* biasI, const float* sink,
                           const int64_t* pos, void* out, void* pool, void* poolI, void* kv_rot,
                           int32_t* idx, void* workspace, size_t ws_bytes, void* stream);

/*
 * One HCA layer in prefill: compress kv -> pool (non-overlapping, rotated) and kv_rot,
 * then attention over every visible entry plus the window.  Requires overlap == 0.
 */
dsv4_status dsv4_hca_layer(const dsv4_params* params, const void* q, const void* kv,
                           const void* z, const float* bias, const float* sink,
                           const int64_t* pos, void* out, void* pool, void* kv_rot,
                           void* workspace, size_t ws_bytes, void* stream);

/*
 * Grouped low-rank output projection ([V4] "Hybrid attention (§2.3)", grouped output
 * projection: o_groups head groups -> o_lora_rank per group (DeepseekV4GroupedLinear,
 * `o_a_proj`) -> hidden_size (`o_b_proj`); no biases).  Head group i holds the contiguous
 * heads [i*H/g, (i+1)*H/g); their outputs, concatenated in head order, are projected by
 * the group's own weight; the g results, concatenated in group order, feed o_b_proj:
 *   u[t, i*dg + r] = sum_c wa[i, r, c] * o[t, i*H/g + c/dv, c % dv]     c < (H/g)*dv
 *   y[t, k]        = sum_j wb[k, j] * u[t, j]                            j < g*dg
 * bf16 in and out, fp32 accumulation on the tensor cores; u is rounded to bf16 between the
 * two products.  Uses H, dv and dtype (must be DSV4_BF16) from params.
 *
 *   T       tokens (rows of o)
 *   groups  o_groups (divides H);  dg  o_lora_rank (a multiple of 256)
 *   hidden  hidden_size (a multiple of 256); (H/groups)*dv must be a multiple of 64
 *   o       [T,H,dv] bf16      attention outputs, read in place
 *   wa      [groups,dg,(H/groups)*dv] bf16   o_a_proj weights (one per group)
 *   wb      [hidden,groups*dg] bf16          o_b_proj weight
 *   u       [T,groups*dg] bf16 out: the grouped intermediate (caller-owned scratch)
 *   y       [T,hidden] bf16    out
 * DSV4_ERR_SHAPE for sizes the kernel does not tile (or dtype float32); validation happens
 * on the host before any launch; allocates nothing.
 */
dsv4_status dsv4_grouped_out_proj(const dsv4_params* params, int32_t T, int32_t groups, int32_t dg,
                                  int32_t hidden, const void* o, const void* wa, const void* wb, void* u,
                                  void* y, void* stream);

/* Bytes of workspace any entry point needs for these params (a pure function of them). */
size_t dsv4_workspace_bytes(const dsv4_params* params);

/* Static, NUL-terminated description of a status code. */
const char* dsv4_status_string(dsv4_status status);

/* Library ABI version (major * 100 + minor). */
int32_t dsv4_version(void);

/* Synchronise `stream`, then read and clear the device-side check words of the current
 * device: DSV4_ERR_DEVICE_CHECK means a kernel gave up a bounded pipeline wait (its CTA
 * returned early and its outputs are invalid), or, with dsv4_set_index_checks on, that an
 * index list was invalid; nothing traps or hangs instead. */
dsv4_status dsv4_device_check(void* stream);

/* Device-side validation of attention index lists ([V4] "Attention mask layout": a query
 * sees entry w only when w < (t+1)/m; empty slots hold -1; each entry is one key).  With
 * the checks on (default: off; on in builds with DSV4_DEBUG), dsv4_sparse_mqa_attn first
 * checks every index list it is given: an entry other than -1 that is negative or not
 * visible sets bit 0 of a device error word, an entry that appears twice in a row sets
 * bit 1 (rows of up to 1,572,864 visible entries; longer rows get the range check only).
 * The attention itself still runs and never reads out of bounds (an entry that is not
 * visible is masked).  dsv4_device_check then returns DSV4_ERR_DEVICE_CHECK and clears the
 * word.  Nothing traps.  The switch is process-wide; it costs one extra launch per call. */
void dsv4_set_index_checks(int32_t on);
int32_t dsv4_index_checks(void);

/* Kernels this process has enqueued through libdsv4 so far (all devices, all entry
 * points); a monotone counter for launch accounting, read without synchronising. */
uint64_t dsv4_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* DSV4_H_ */
