/*
 * speckv.h -- C ABI of the B200 (sm_100a) lookahead importance-scoring library.
 *
 * The method is "Draft-based Approximate Inference for LLMs" (paper notes,
 * ICLR 2026, arXiv 2506.08373):
 *   - section 关键设计, SpecKV: for every attention head, the queries of the
 *     last n_window input tokens and of the n_lookahead draft (lookahead)
 *     tokens attend to the input keys; the attention that the remaining input
 *     keys receive estimates the importance of each KV pair; the top-C_max KV
 *     pairs plus the window are kept.
 *   - section 关键设计, SpecPC: draft attention A[layer][head][query][key] over
 *     a large query window with weights that fall with distance from the end,
 *     the first l_skip layers skipped, averaged first, then maximised.
 *   - section 关键设计, SpecKV-PC: SpecPC first, then SpecKV on what it kept.
 *   - section 损失函数 / 训练策略: SpecPC smooths scores with local pooling.
 *
 * Conventions for every entry point
 *   - Tensor arguments are DEVICE pointers owned by the caller, contiguous in
 *     the layouts given below, 16-byte aligned.  The library allocates no
 *     memory: scratch space is the caller's `workspace`, whose size comes from
 *     the matching *_workspace_size() query.
 *   - bf16 means IEEE bfloat16 bit patterns (uint16_t); fp32 is float.
 *   - All work is enqueued on `stream` (a cudaStream_t, passed as void*;
 *     NULL = legacy default stream) and returns without host synchronisation.
 *   - The return value is a spk_status.  Argument errors are detected on the
 *     host and returned BEFORE anything is launched; spk_last_error() then
 *     describes the problem (thread-local string).
 *   - Errors found on the device (a bounded wait that timed out, an index
 *     outside its range in kv_compact) are recorded in device error words
 *     that spk_device_error() reads; kernels never trap.
 *   - Results are deterministic: the same inputs give bitwise identical
 *     outputs (no floating-point atomics).
 *   - Calls on the same stream are ordered; calls that share a workspace must
 *     not run concurrently on different streams.
 */
#ifndef SPECKV_H
#define SPECKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SPK_OK = 0,
  SPK_ERR_ARG = 1,          /* a null/misaligned pointer or an inconsistent shape */
  SPK_ERR_UNSUPPORTED = 2,  /* a valid shape outside what the kernels implement */
  SPK_ERR_WORKSPACE = 3,    /* workspace missing or smaller than *_workspace_size() */
  SPK_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed (see spk_last_error) */
  SPK_ERR_TIMEOUT = 5       /* reported by spk_device_error: a device wait ran out */
} spk_status;

/* ------------------------------------------------------------------------
 * SpecKV scoring (section 关键设计, SpecKV)
 *
 * A unit is one (batch element, layer, KV head); units are numbered
 * u = (b * layers + l) * hkv + h.  Query head qh belongs to KV head qh / g,
 * g = hq / hkv (GQA).  R = n_window + n_lookahead query rows per query head:
 * row i < n_window is the window query at input position n_in - n_window + i
 * and sees input keys 0 .. n_in - n_window + i (causal); row i >= n_window is
 * a lookahead (draft) query and sees all n_in input keys.  Keys of the
 * lookahead tokens are not input keys and are not part of the softmax.
 *
 *   q      bf16 [batch][layers][hq][R][head_dim]   (rows pre-scaled or not: see scale)
 *   k      bf16 [batch][layers][hkv][n_in][head_dim]
 *   scores fp32 [units][n_pre], n_pre = n_in - n_window:
 *          scores[u][j] = sum over the g query heads of unit u and their R rows
 *                         of softmax_j(scale * q_row . k_j)   (prefix keys only)
 *   window_mass fp32 [units][n_window] or NULL: the same sum on the window keys
 *          j = n_pre .. n_in-1 (every prefix and window column together sum to
 *          g * R per unit, which makes it a conservation check).
 *
 * Supported: head_dim in {64, 128}; hq % hkv == 0; g * R <= 2048;
 * 0 <= n_window <= n_in; R >= 1; scale > 0 and finite.
 * ------------------------------------------------------------------------ */
typedef struct {
  int batch, layers, hq, hkv, head_dim;
  int n_in, n_window, n_lookahead;
  float scale; /* multiplies q.k before the softmax (1.0 if q is pre-scaled) */
} spk_speckv_shape;

/* Workspace: the row offsets pass 1 hands to pass 2, 32 bytes per query row
 * with each unit's g * R rows rounded up to 128:
 * units * ceil(g * R / 128) * 4096 bytes (rounded up to 256); 16-byte aligned. */
size_t speckv_workspace_size(const spk_speckv_shape* shape);

spk_status speckv_score(const spk_speckv_shape* shape, const void* q_bf16, const void* k_bf16,
                        float* scores, float* window_mass, void* workspace, size_t workspace_bytes,
                        void* stream);

/* The two passes of speckv_score as separate calls, for callers that time
 * or schedule them apart; speckv_score is exactly speckv_row_offsets
 * followed by speckv_colsum on the same stream.
 *   speckv_row_offsets: pass 1 -- every query row's log-sum-exp, stored in the
 *     workspace as the row offsets pass 2 adds to its logits;
 *   speckv_colsum: pass 2 -- the scores (and window mass) from a workspace that
 *     speckv_row_offsets filled for the same shape, q and k (ordered before
 *     this call; the workspace is only read).
 * Same shapes, layouts, workspace size and rules as speckv_score. */
spk_status speckv_row_offsets(const spk_speckv_shape* shape, const void* q_bf16, const void* k_bf16,
                              void* workspace, size_t workspace_bytes, void* stream);

spk_status speckv_colsum(const spk_speckv_shape* shape, const void* q_bf16, const void* k_bf16, float* scores,
                         float* window_mass, const void* workspace, size_t workspace_bytes, void* stream);

/* Pass 1 alone (diagnostic): the log2-domain log-sum-exp of every query row,
 * lse2[u][qh_local * R + i] = log2 sum_{visible j} 2^(scale*log2(e) * q.k_j),
 * fp32 [units][g * R].  Same shapes and rules as speckv_score. */
spk_status speckv_row_lse(const spk_speckv_shape* shape, const void* q_bf16, const void* k_bf16,
                          float* lse2, void* stream);

/* speckv_score for callers that cannot allocate device memory.  The paper
 * has no counterpart: this is a deployment variant.  Serving engines that
 * reserve nearly all of HBM for their own KV-cache pool, and plugin hosts
 * that give plugins no access to the CUDA allocator, can neither cudaMalloc
 * nor spare a workspace; this call keeps pass 1's row offsets in a fixed
 * 16 MiB array inside the library image instead (no allocation of any kind).
 *   - Same shapes, layouts, outputs and rules as speckv_score.
 *   - Rejects (SPK_ERR_UNSUPPORTED, before any launch) shapes whose workspace
 *     (speckv_workspace_size) would exceed 16 MiB, i.e. more than 524,288
 *     query rows with each unit's rows rounded up to 128.
 *   - Every GPU that loads the library holds the 16 MiB until process exit.
 *   - The first call on a device looks up the array's address on that device
 *     (cudaGetSymbolAddress) and caches it: make it before any stream capture.
 *     A cudaDeviceReset unloads the library's device image, so the cached
 *     address is stale afterwards: do not call this entry point again in a
 *     process that has reset the device.
 *   - All calls share the array, which keeps the last call's contents (every
 *     entry read is first rewritten by the same call, so nothing needs
 *     clearing); calls whose kernels overlap on the GPU race on it. */
spk_status speckv_score_static_ws(const spk_speckv_shape* shape, const void* q_bf16, const void* k_bf16,
                                  float* scores, float* window_mass, void* stream);

/* ------------------------------------------------------------------------
 * Prefill attention of the window and lookahead rows (section 关键设计,
 * SpecKV: the input tokens and the lookahead tokens go through the target
 * model's prefill together, and the importance scores are read from the
 * attention of the last n_window input rows and of the lookahead rows)
 *
 * The key/value sequence of a unit is its n_in input tokens followed by its
 * n_lookahead lookahead tokens.  Query row i of a head (R = n_window +
 * n_lookahead rows, ordered as for speckv_score) sits at position
 * n_in - n_window + i and attends causally to the keys up to that position:
 *   out[u][row]   = softmax_j(scale * q_row . k_j) . v_j over those keys
 *   lse2[u][row]  = log2 sum_{j < min(pos + 1, n_in)} 2^(scale*log2(e) * q_row . k_j)
 *                   -- the same input-key normaliser as speckv_row_lse
 *   workspace     = (when non-NULL) the row offsets exactly as
 *                   speckv_row_offsets writes them, so that speckv_colsum on
 *                   the same shape, q and k gives the importance scores
 *                   without the scoring's own first pass.
 *
 *   q              bf16 [batch][layers][hq][R][head_dim]
 *   k, v           bf16 [batch][layers][hkv][n_in][head_dim]         (input tokens)
 *   k_look, v_look bf16 [batch][layers][hkv][n_lookahead][head_dim]  (NULL if n_lookahead = 0)
 *   out            bf16 [batch][layers][hq][R][head_dim]
 *   lse2           fp32 [units][g * R] or NULL
 *   workspace      NULL, or speckv_workspace_size(shape) bytes, 16-byte aligned
 * Probabilities enter the P.V product as bf16 (fp32 accumulation); the
 * normaliser and lse2 are formed from the fp32 probabilities.
 * Supported: as speckv_score.
 * ------------------------------------------------------------------------ */
spk_status speckv_prefill_attention(const spk_speckv_shape* shape, const void* q_bf16, const void* k_bf16,
                                   const void* v_bf16, const void* k_look_bf16, const void* v_look_bf16,
                                   void* out_bf16, float* lse2, void* workspace, size_t workspace_bytes,
                                   void* stream);

/* ------------------------------------------------------------------------
 * Vertical-Slash sparse prefill attention (section 损失函数 / 训练策略: SpecKV
 * runs the target prefill with Vertical-Slash sparse attention, the pattern
 * of the cited sparse-attention work)
 *
 * Per unit (batch element, layer, KV head) the pattern is a set of vertical
 * key columns and a set of slash diagonals (offsets o = p - j).  The query
 * row at position p attends to the keys j <= p with j in vertical, or
 * p - j in slash, or j = p (a token always sees itself):
 *   out[u*g + h][i] = softmax_j(scale * q . k_j) . v_j over those keys,
 *   lse2[u*g + h][i] = log2 sum_j 2^(scale*log2(e) * q . k_j)   (optional)
 * Query rows are the last n_q positions: row i sits at n - n_q + i.
 *
 *   q         bf16 [batch][layers][hq][n_q][head_dim]
 *   k, v      bf16 [batch][layers][hkv][n][head_dim]
 *   vertical  int32 [units][n_vertical], ascending, unique, in [0, n)
 *   slash     int32 [units][n_slash], ascending, unique, in [0, n)
 *   out       bf16 [batch][layers][hq][n_q][head_dim]
 *   lse2      fp32 [units * g][n_q] or NULL
 *   workspace vs_workspace_size(shape) bytes (the vertical keys' K and V rows,
 *             gathered on the stream first), 16-byte aligned; may be NULL when
 *             n_vertical = 0
 * A vertical or slash entry outside [0, n) is ignored and recorded as
 * SPK_ERR_ARG in the device error word; unsorted lists give wrong results.
 * Probabilities enter the P.V product as bf16 (fp32 accumulation).
 * Supported: head_dim in {64, 128}; hq % hkv == 0; 1 <= n_q <= n <= 65536;
 * n_vertical <= 4096; n_slash <= n.
 * ------------------------------------------------------------------------ */
typedef struct {
  int batch, layers, hq, hkv, head_dim;
  int n, n_q, n_vertical, n_slash;
  float scale;
} spk_vs_shape;

size_t vs_workspace_size(const spk_vs_shape* shape);

spk_status vs_sparse_attention(const spk_vs_shape* shape, const void* q_bf16, const void* k_bf16,
                               const void* v_bf16, const int32_t* vertical, const int32_t* slash, void* out_bf16,
                               float* lse2, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * SpecPC scoring (section 关键设计, SpecPC)
 *
 * Per batch element b, the draft's last W = n_rows query positions: row i sits
 * at position n_in + n_lookahead - 1 - W + i and sees input keys 0 .. that
 * position (capped at n_in - 1).  For every query head qh and layer
 * l >= l_skip, P[l][qh][i][j] is the causal softmax of scale * q . k_j.
 *   S[qh][j] = ( sum_{l >= l_skip} sum_i w_i P[l][qh][i][j] ) / ( sum_i w_i * (layers - l_skip) )
 *   scores[b][j] = max_qh S[qh][j]        for j in 0 .. n_in-1
 *
 *   q            bf16 [batch][layers][hq][W][head_dim]   (layers < l_skip are not read)
 *   k            bf16 [batch][layers][hkv][n_in][head_dim]
 *   row_weights  fp32 [W], device, oldest row first, w_i >= 0, sum > 0; a row
 *                of weight 0 contributes nothing (its attention is not read)
 *   scores       fp32 [batch][n_in]
 *
 * Supported: head_dim in {64, 128}; hq % hkv == 0; hq <= 32; (hq/hkv) * W <= 2048;
 * 0 <= l_skip < layers; 1 <= W <= n_in + n_lookahead - 1; n_lookahead >= 1.
 * ------------------------------------------------------------------------ */
typedef struct {
  int batch, layers, l_skip, hq, hkv, head_dim;
  int n_in, n_rows, n_lookahead;
  float scale;
} spk_specpc_shape;

/* Workspace: the row offsets, units * ceil((hq/hkv) * W / 128) * 4096 bytes
 * (rounded up to 256), units = batch * (layers - l_skip) * hkv; when the
 * column pass would leave SMs of the current device idle (few 256-key blocks,
 * e.g. batch 1 at 32K), it splits each block's (KV head, layer) segments into
 * G groups (G <= 16, chosen from the device's SM count) and adds
 * batch * ceil(n_in / 256) * G * hq * 1 KB of per-head partial sums, which a
 * merge kernel adds in a fixed order (results stay bitwise reproducible on a
 * given device).  Query the size with the device current; 16-byte aligned. */
size_t specpc_workspace_size(const spk_specpc_shape* shape);

spk_status specpc_score(const spk_specpc_shape* shape, const void* q_bf16, const void* k_bf16,
                        const float* row_weights, float* scores, void* workspace, size_t workspace_bytes,
                        void* stream);

/* The two passes of specpc_score as separate calls (specpc_score is exactly
 * specpc_row_offsets followed by specpc_colsum on the same stream): the row
 * offsets with the row weights folded in, then the scores from them. */
spk_status specpc_row_offsets(const spk_specpc_shape* shape, const void* q_bf16, const void* k_bf16,
                              const float* row_weights, void* workspace, size_t workspace_bytes, void* stream);

spk_status specpc_colsum(const spk_specpc_shape* shape, const void* q_bf16, const void* k_bf16, float* scores,
                         void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Pooling + top-k selection (section 关键设计: keep the top-C_max KV pairs plus
 * the window; section 损失函数 / 训练策略: local pooling keeps token runs)
 *
 * For each of `units` rows of n_cand candidate scores, r = pool_kernel / 2 and
 * W_j = [j - r, j + r] ∩ [0, n_cand) (the window clipped at the row's ends):
 *   pooled[j] = max of scores over W_j                 (SPK_POOL_MAX)
 *             = (sum of scores over W_j) / |W_j|       (SPK_POOL_AVG; fp32, summed
 *               in index order, one correctly rounded division)
 *   selected  = the min(k, n_cand) largest pooled values; equal values are
 *               taken lowest index first
 *   idx[u]    = selected indices in ascending order, then the tail
 *               n_cand, n_cand + 1, .., n_cand + n_tail - 1 (the kept window)
 *
 *   scores  fp32 [units][n_cand], finite (NaN order is unspecified; -0 == +0)
 *   idx     int32 [units][min(k, n_cand) + n_tail]
 *   pooled  fp32 [units][n_cand] or NULL
 *
 * The pages say "local pooling" without its kind; the workloads use max
 * pooling, which is what topk_select does.  topk_select_pool takes the mode.
 * Workspace: units * round_up(n_cand, 4) * 4 bytes, 16-byte aligned (the
 * order-preserving 32-bit keys of the pooled values, one padded row per
 * unit).  It is required by the contract; rows of up to 327,680 candidates
 * with pool_kernel <= 2049 keep their keys in shared memory instead and
 * leave it untouched.
 *
 * Supported: pool_kernel odd >= 1; k >= 0; n_tail >= 0; n_cand >= 0;
 * pool_mode SPK_POOL_MAX or SPK_POOL_AVG.
 * ------------------------------------------------------------------------ */
typedef enum {
  SPK_POOL_MAX = 0,
  SPK_POOL_AVG = 1
} spk_pool_mode;

size_t topk_workspace_size(int units, int n_cand);

spk_status topk_select(const float* scores, int units, int n_cand, int pool_kernel, int k, int n_tail,
                       int32_t* idx, float* pooled, void* workspace, size_t workspace_bytes, void* stream);

spk_status topk_select_pool(const float* scores, int units, int n_cand, int pool_mode, int pool_kernel, int k,
                            int n_tail, int32_t* idx, float* pooled, void* workspace, size_t workspace_bytes,
                            void* stream);

/* ------------------------------------------------------------------------
 * KV compaction (section 关键设计, SpecKV: the dropped cache keeps only the
 * selected KV pairs)
 *
 *   k_out[u][t] = k[u][ idx[u / units_per_idx][t] ],  same for v
 *   k, v         [units][n_src][head_dim] elements of elem_bytes bytes
 *   idx          int32 [units / units_per_idx][n_idx], each in [0, n_src)
 *   k_out, v_out [units][n_idx][head_dim]
 * units_per_idx = 1 gives every unit its own index row; units_per_idx =
 * layers * hkv shares one row across all (layer, KV head) of a batch element
 * (SpecPC / SpecKV-PC).  v and v_out may both be NULL.  Rows are copied
 * byte for byte.  An index outside [0, n_src) leaves that output row
 * unwritten and records SPK_ERR_ARG in the device error word.  k and v may
 * be device addresses of pinned host memory (spk_mapped_host_pointer): only
 * the selected rows are then read over the host link.
 *
 * Supported: head_dim * elem_bytes a multiple of 16; units % units_per_idx == 0.
 * ------------------------------------------------------------------------ */
spk_status kv_compact(const void* k, const void* v, int units, int n_src, int head_dim, int elem_bytes,
                      const int32_t* idx, int n_idx, int units_per_idx, void* k_out, void* v_out,
                      void* stream);

/* ------------------------------------------------------------------------
 * Decode attention over a compacted cache (section 整体框架: the target model
 * then runs on the compressed KV cache; section 关键设计, SpecKV: the cache
 * holds the kept KV pairs).  One new query token per attention head:
 *
 *   out[b][l][qh][:] = sum_t softmax_t(scale * q[b][l][qh] . k[b][l][qh/g][t]) * v[b][l][qh/g][t]
 *   q      bf16 [batch][layers][hq][head_dim]
 *   k, v   bf16 [batch][layers][hkv][n_kv][head_dim]   (e.g. kv_compact's outputs)
 *   out    fp32 [batch][layers][hq][head_dim]
 * The softmax runs over all n_kv rows (the caller appends the new token's own
 * K/V row when it should attend to itself).  Deterministic.
 *
 * Supported: head_dim in {64, 128}; hq % hkv == 0; hq / hkv <= 8; n_kv >= 1;
 * scale > 0 and finite.
 * ------------------------------------------------------------------------ */
spk_status decode_attention(int batch, int layers, int hq, int hkv, int head_dim, int n_kv, float scale,
                            const void* q_bf16, const void* k_bf16, const void* v_bf16, float* out,
                            void* stream);

/* Device address of page-locked, device-mapped host memory (a deployment
 * helper; the paper has no counterpart).  k and v of kv_compact may point
 * into such memory: the gather then reads only the selected rows over the
 * host link instead of copying the whole cache to the device first.
 *   host  a pointer into memory from cudaHostAlloc / cudaHostRegister (any
 *         offset into the allocation)
 *   *dev  the address kernels use for it (owned by the caller's allocation)
 * Returns SPK_ERR_CUDA (and leaves *dev untouched) when the memory is not
 * page-locked and mapped, or no device is present. */
spk_status spk_mapped_host_pointer(const void* host, void** dev);

/* ------------------------------------------------------------------------
 * Errors
 * ------------------------------------------------------------------------ */
/* Message for the last non-OK status returned on this thread ("" if none). */
const char* spk_last_error(void);

/* Synchronises the current device, then reports an error recorded by a
 * kernel since the last clear: *status = SPK_OK, SPK_ERR_TIMEOUT (a bounded
 * device wait ran out; *site says where) or SPK_ERR_ARG (an index out of
 * range in kv_compact or vs_sparse_attention).  Each source file of the
 * library keeps its own first-error word; the first set one, in a fixed
 * order of the files, is reported.  clear != 0 resets them all.  Returns
 * SPK_ERR_CUDA if the device could not be read. */
spk_status spk_device_error(int* status, int* site, int clear);

/* Diagnostic: y[i] = 2^t[i] as computed on the FMA pipe by the scoring
 * epilogues (range reduction + fitted degree-4 polynomial, relative error
 * <= 2.7e-6 for t in [-126, 64); arguments below -126 give a value under
 * 1.2e-38).  t, y: fp32 device arrays of n elements. */
spk_status spk_exp2_fma(const float* t, float* y, int n, void* stream);

/* Self-test of the bounded waits: launches one kernel that waits on a barrier
 * nothing will complete, with a limit of limit_ns nanoseconds (clamped to
 * [1e3, 1e9]).  The kernel gives up, records SPK_ERR_TIMEOUT at site 999 and
 * returns; read it with spk_device_error().  No GPU state is left behind. */
spk_status spk_selftest_wait_timeout(long long limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SPECKV_H */
