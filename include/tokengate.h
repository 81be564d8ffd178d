/*
 * tokengate.h -- C ABI of the TokenGate prefill hot path on NVIDIA B200 (sm_100a).
 *
 * The calls implement, as CUDA kernels, the gate layer and the token-gated attention
 * described on these pages (cited below by tag, with the section used):
 *   [fluxbbs]    "TokenGate 长上下文预填充提速 11.3 倍，斯坦福伯克利开源门控剪枝"
 *   [digest]     "TokenGate: Adapting LLMs for Fast and Memory-Efficient Prefill with
 *                 Learned Token Pruning" (paper digest)
 *   [farwalk]    "斯坦福与 UC Berkeley 提出 TokenGate：token 门控注意力让长上下文预填充最高快 11.3 倍"
 *   [aiwillknow] "TokenGate：让模型学会跳读，而不只压缩 KV 缓存"
 *
 * Conventions shared by every call
 *   - Pointers are device pointers unless the name ends in `_host`.  The caller owns
 *     every buffer; unless an entry point says otherwise, the library allocates no
 *     device memory.  Scratch memory is passed in as `workspace`, sized by the
 *     matching *_workspace_size() query.
 *   - Matrices are row-major; `ld_*` is the row stride in elements.  bf16 tensors are
 *     passed as their 16-bit patterns (tg_bf16).
 *   - Requests are packed back to back ("varlen"): request b owns rows
 *     cu_seqlens[b] .. cu_seqlens[b+1]-1 before the gate and kept rows
 *     cu_kept[b] .. cu_kept[b+1]-1 after it.  Each cu array is given twice: on the
 *     device (read by kernels) and on the host (argument checks and launch shapes);
 *     the two copies must hold the same values.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and never synchronises, except tg_status_read().
 *   - Return value: TG_OK, or a negative TG_ERR_* code.  Argument errors are found on
 *     the host before anything is launched.  Errors found on the device (a bounded
 *     wait that ran out, a kept count that disagrees with the prunable mask) are
 *     OR-ed into the caller's 32-bit `status` word (TG_STATUS_* bits); read it with
 *     tg_status_read().  `status` may be NULL where a call says so.
 *   - Device requirement: compute capability 10.0 (B200).  Other devices get
 *     TG_ERR_UNSUPPORTED_DEVICE; there is no fallback path.
 */
#ifndef TOKENGATE_H
#define TOKENGATE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t tg_bf16;   /* bfloat16 bit pattern */
typedef void* tg_stream_t;  /* cudaStream_t */

/* Return codes. */
#define TG_OK 0
#define TG_ERR_INVALID_ARGUMENT (-1)   /* null pointer, bad size, inconsistent cu arrays */
#define TG_ERR_MISALIGNED (-2)         /* pointer or row stride not 16-byte aligned */
#define TG_ERR_UNSUPPORTED_DEVICE (-3) /* current device is not sm_100 */
#define TG_ERR_WORKSPACE (-4)          /* workspace missing or smaller than required */
#define TG_ERR_CUDA (-5)               /* a CUDA runtime/driver call failed; see tg_last_cuda_error */
#define TG_ERR_UNSUPPORTED_SHAPE (-6)  /* a dimension outside what the kernels implement */
#define TG_ERR_SCRATCH_LIMIT (-7)      /* larger than the fixed scratch of tg_gate_score_noalloc */

/* Device status bits (OR-ed into the caller's status word by kernels). */
#define TG_STATUS_TIMEOUT 0x1u /* a bounded wait ran out; outputs of that call are invalid */
#define TG_STATUS_BUDGET 0x2u  /* kept count K_b inconsistent with the prunable mask */
#define TG_STATUS_BOUNDS 0x4u  /* a row index outside the source; that row was skipped */
#define TG_STATUS_WORKSPACE 0x8u /* a split-attention workspace was not zero-filled */

/* ------------------------------------------------------------------ utilities */

/* Short English description of a TG_* return code (static storage). */
const char* tg_error_string(int code);

/* cudaError_t value behind the most recent TG_ERR_CUDA on the calling thread. */
int tg_last_cuda_error(void);

/* 1 if `device` is a compute-capability-10.0 GPU this library runs on, else 0. */
int tg_device_supported(int device);

/* Library ABI version (major * 100 + minor). */
int tg_version(void);

/* Zero the status word (async on `stream`). */
int tg_status_clear(uint32_t* status, tg_stream_t stream);

/* Copy the status word to *out_host after synchronising `stream`. */
int tg_status_read(const uint32_t* status, uint32_t* out_host, tg_stream_t stream);

/* Launch overlap (library-wide, default on; not part of the method).  When on, every
 * kernel of this library is launched with CUDA programmatic stream serialisation: it
 * may start once the kernel before it on the stream has retired all its thread
 * blocks, or earlier when that kernel is the CTA-pair GEMM, which lets the next kernel
 * in as soon as all its own thread blocks are past their dependency wait (they are all
 * resident: one wave); the next kernel's blocks then take only free SMs.  A kernel
 * started this way runs only set-up work that touches no caller memory (barriers,
 * tensor memory) and waits for the earlier kernel to complete before it reads or
 * writes any buffer.  Results are identical either way.  The 16k gated step (CUDA
 * graph) runs 2.5% faster with it on, the 128k step the same.  The setting is read at
 * each launch; the caller orders changes with its own launches.
 * tg_set_launch_overlap: enable = 0 turns it off, anything else on; returns TG_OK.
 * tg_get_launch_overlap: the current setting (0 or 1). */
int tg_set_launch_overlap(int enable);
int tg_get_launch_overlap(void);

/* Which kernel serves the gather mode of tg_gather_rope (no RoPE).  Off (the default):
 * one warp per row with 16-byte loads and stores, every row of a batch loaded before it
 * is stored.  On: the TMA row gather (tile::gather4 loads of four kept rows at a time,
 * tiled TMA stores of four consecutive destination rows), used when width is a multiple
 * of 64 and at most 8192 and the row counts fit in int32.  Both write the same bytes and
 * report out-of-range indices the same way; on B200 the warp-per-row copy measured
 * faster at the kept-row counts of the 16k and 128k steps.  Read at each call.
 * tg_set_gather_tma: enable = 0 selects the warp-per-row copy; returns TG_OK.
 * tg_get_gather_tma: the current setting (0 or 1). */
int tg_set_gather_tma(int enable);
int tg_get_gather_tma(void);

/* Which kernel runs the scorer GEMM of tg_gate_score (and tg_gate_score_noalloc).  On
 * (the default): persistent CTA pairs over 256-row tiles (tcgen05 cta_group::2, each CTA
 * streaming half of W1 per k-block, two accumulators so a tile's epilogue overlaps the
 * next tile's loads); off: one CTA per 128-row tile.  Both form the same products in the
 * same order, so s, z and bias are identical.  Read at each call.
 * tg_set_scorer_pair: enable = 0 selects the one-CTA kernel; returns TG_OK.
 * tg_get_scorer_pair: the current setting (0 or 1). */
int tg_set_scorer_pair(int enable);
int tg_get_scorer_pair(void);

/* L2 prefetch hint (not part of the method): issue bulk prefetches that bring
 * [ptr, ptr + bytes) into the L2 cache ahead of a later kernel that reads it (the
 * next layer's weights while attention runs, for instance).  Nothing waits for the
 * data and results never depend on it.  ptr 16-byte aligned; bytes is rounded down to a
 * multiple of 16 (0 does nothing).  Asynchronous on `stream`; one small kernel launch. */
int tg_prefetch_l2(const void* ptr, size_t bytes, tg_stream_t stream);

/*
 * Rotary table for original-position RoPE ([aiwillknow] figure 1(a)(b): kept tokens
 * keep their original position encoding).  Writes cos_sin[p][i][0] = cos(p * f_i),
 * cos_sin[p][i][1] = sin(p * f_i) for p < max_pos, i < head_dim/2, with
 * f_i = theta^(-2 i / head_dim).  Angles and trigonometry are evaluated in float64
 * on the device, then rounded to float32.  cos_sin: float32 [max_pos, head_dim/2, 2].
 */
int tg_rope_table(float* cos_sin, int max_pos, int head_dim, double theta,
                  tg_stream_t stream);

/*
 * Per-row rotary table (same source: every kept row rotates by its original position).
 * Copies each row's row of the tg_rope_table table, transposed in 16-byte blocks so that
 * block j of consecutive rows is contiguous:
 *   rot[(j * ld_rot + r) * 4 + e] = cos_sin[pos[r] * head_dim + 4 j + e],  e < 4,
 * for r < n_rows, j < head_dim / 4 (block j holds cos, sin of rotation pairs 2j, 2j + 1).
 * Passed to the QKV entry points with pos = NULL (cos_sin = rot, max_pos = ld_rot), it
 * gives the same results as (pos, cos_sin) with contiguous table reads in the GEMM
 * epilogue; the kept positions are the same in every gated layer, so one call per step
 * serves all of them.  pos: int32 [n_rows] (values < max_pos, else TG_STATUS_BOUNDS and
 * the row takes position 0); cos_sin: float32 [max_pos, head_dim] (16-byte aligned);
 * rot: float32 [head_dim / 4, ld_rot, 4] (16-byte aligned), ld_rot >= n_rows; head_dim a
 * multiple of 4 (>= 8).  status may be NULL.  Not a step of the method: a layout change.
 */
int tg_rope_rows(const int32_t* pos, int64_t n_rows, const float* cos_sin, int max_pos,
                 int head_dim, float* rot, int64_t ld_rot, uint32_t* status,
                 tg_stream_t stream);

/*
 * Host-only planning of the kept counts from per-request budgets (no GPU work).
 * ([farwalk] How do you deploy TokenGate?: generation takes a budget of kept prefill
 *  tokens; [farwalk] How does TokenGate learned token pruning work?: the question is
 *  never pruned.)  The budget counts every kept token, question included:
 *    K_b = Q_b + min(D_b, max(0, budget_b - Q_b)),  D_b = N_b - Q_b,
 * so a budget below Q_b keeps the question only and one above N_b keeps everything.
 * cu_seqlens_host int32 [batch+1]; n_question_host int32 [batch] (Q_b, non-prunable
 * tokens of request b); budgets_host int32 [batch]; writes cu_kept_host int32 [batch+1].
 */
int tg_plan_kept(const int32_t* cu_seqlens_host, const int32_t* n_question_host,
                 const int32_t* budgets_host, int batch, int32_t* cu_kept_host);

/* ------------------------------------------------------------------ gate scoring */

/* Bytes of workspace tg_gate_score needs for `total_tokens` rows and `batch` requests. */
size_t tg_gate_score_workspace_size(int64_t total_tokens, int hidden, int width, int batch);

/*
 * Gate scores and their sequence normalisation
 * ([fluxbbs] 门控到底插在模型的哪个位置: a small MLP scores each token's normalised
 *  residual and the scores are RMSNorm-normalised along the sequence;
 *  [farwalk] How does TokenGate learned token pruning work?: the residual is the
 *  post-attention residual at the gate layer).
 *
 *   x_t    = h_t * norm_w / sqrt(mean(h_t^2) + eps_norm)
 *   s_t    = sum_f w2[f] * SiLU((W1 x_t)[f])
 *   z_t    = s_t / sqrt(mean_{t' in request(t)} s_t'^2 + eps_seq)
 *   bias_t = z_t if prunable[t] else 0
 *
 * h:        bf16 [total_tokens, hidden], row stride ld_h (multiple of 8).
 * norm_w:   float32 [hidden] RMSNorm weight, or NULL for all ones.  When given it is
 *           folded into W1 (rounded to bf16) inside the workspace.
 * W1:       bf16 [width, hidden] (output rows), row stride hidden.  width must be 256.
 * w2:       float32 [width].
 * cu_seqlens / cu_seqlens_host: int32 [batch+1], cu_seqlens[batch] = total_tokens.
 * prunable: uint8 [total_tokens], 1 = document (prunable), 0 = question (kept).
 * s_out, z_out, bias_out: float32 [total_tokens] (any of them may alias nothing else).
 * hidden must be a multiple of 64.  status may be NULL.
 * The GEMM runs on tcgen05 tensor cores with the row RMS applied in its epilogue and
 * per-32-row partial sums of s^2 written there; a second kernel reduces the partials
 * of each request in a fixed order (bit-reproducible) and writes z and bias.
 */
int tg_gate_score(const tg_bf16* h, int64_t ld_h, int64_t total_tokens, int hidden,
                  const float* norm_w, const tg_bf16* W1, int width, const float* w2,
                  float eps_norm, const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
                  int batch, float eps_seq, const uint8_t* prunable, float* s_out,
                  float* z_out, float* bias_out, void* workspace, size_t workspace_bytes,
                  uint32_t* status, tg_stream_t stream);

/*
 * Sequence RMSNorm of raw scores on its own ([fluxbbs] 门控到底插在模型的哪个位置):
 *   z_t = s_t / sqrt(mean_{t' in request(t)} s_t'^2 + eps_seq),  bias_t = prunable ? z_t : 0.
 * Same kernel and fixed reduction order as the second stage of tg_gate_score, reading
 * s directly instead of per-chunk partial sums.  s, z_out, bias_out float32 [total];
 * z_out and bias_out must not alias s.  No workspace.
 */
int tg_seq_rmsnorm(const float* s, const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
                   int batch, const uint8_t* prunable, float eps_seq, float* z_out,
                   float* bias_out, tg_stream_t stream);

/*
 * tg_gate_score without a workspace argument, for callers that cannot allocate device
 * memory (for example a serving engine that plans all device memory ahead and forbids
 * allocation during a request, a plug-in limited to the buffers its host framework
 * hands it, or a path that cannot afford cudaMalloc's implicit device synchronisation).
 * The pages have no counterpart of this call: it is a deployment convenience only.
 * Same arguments, results and errors as tg_gate_score, minus workspace/workspace_bytes.
 * Scratch comes from one array compiled into the library (about 2.2 MB), which every GPU
 * that loads the library keeps until the process exits.  Limits: total_tokens <=
 * TG_NOALLOC_MAX_TOKENS and hidden <= TG_NOALLOC_MAX_HIDDEN, else TG_ERR_SCRATCH_LIMIT
 * and nothing is launched.  The first call on each device looks up the array's device
 * address (cudaGetSymbolAddress); make that first call before any stream capture.  All
 * calls share the one array: calls whose GPU work can overlap (different streams, or
 * several host threads) race on it, so serialise them.  The library allocates nothing
 * here (no cudaMalloc/cudaFree, no allocating library routine).
 */
#define TG_NOALLOC_MAX_TOKENS (1 << 20)
#define TG_NOALLOC_MAX_HIDDEN 4096
int tg_gate_score_noalloc(const tg_bf16* h, int64_t ld_h, int64_t total_tokens, int hidden,
                          const float* norm_w, const tg_bf16* W1, int width, const float* w2,
                          float eps_norm, const int32_t* cu_seqlens,
                          const int32_t* cu_seqlens_host, int batch, float eps_seq,
                          const uint8_t* prunable, float* s_out, float* z_out,
                          float* bias_out, uint32_t* status, tg_stream_t stream);

/* ------------------------------------------------------------------ selection */

/*
 * Prunable-only top-K with order-preserving compaction
 * ([fluxbbs] 门控到底插在模型的哪个位置: keep the top-K tokens, the question is never
 *  pruned; [farwalk] How does TokenGate learned token pruning work?: only the document
 *  is prunable; [aiwillknow] figure 1(a)(b): kept tokens keep their positions).
 *
 * For request b with Q_b non-prunable tokens and K_b = cu_kept[b+1] - cu_kept[b]
 * kept rows, the Kd_b = K_b - Q_b prunable tokens with the largest z are kept, ties
 * going to the lower index; NaN ranks below every number and -0 equals +0.  All
 * non-prunable tokens are kept.  Kept tokens are listed by ascending position:
 *   kept_idx[cu_kept[b] + r]  = cu_seqlens[b] + j   (packed row id of the token)
 *   kept_pos[cu_kept[b] + r]  = j                   (position inside the request)
 *   kept_bias[cu_kept[b] + r] = z[cu_seqlens[b] + j] if prunable, else 0
 * The caller derives cu_kept from its budgets, e.g. K_b = Q_b + min(D_b, max(0,
 * budget_b - Q_b)); if some K_b does not satisfy Q_b <= K_b <= N_b on the device,
 * that request's outputs are left unwritten and TG_STATUS_BUDGET is set.
 * z: float32 [total_tokens]; prunable: uint8 [total_tokens];
 * kept_idx, kept_pos: int32 [cu_kept[batch]]; kept_bias: float32 [cu_kept[batch]].
 * One thread-block cluster per request runs a 3-pass radix select (11/11/10 bits)
 * over order-preserving integer keys with the histograms exchanged through
 * distributed shared memory, then compacts with warp ballots.  status may be NULL.
 */
int tg_topk_compact(const float* z, const uint8_t* prunable, const int32_t* cu_seqlens,
                    const int32_t* cu_seqlens_host, const int32_t* cu_kept,
                    const int32_t* cu_kept_host, int batch, int32_t* kept_idx,
                    int32_t* kept_pos, float* kept_bias, uint32_t* status,
                    tg_stream_t stream);

/* ------------------------------------------------------------------ gather / RoPE */

/*
 * Row gather with optional rotary embedding at original positions
 * ([fluxbbs] 门控到底插在模型的哪个位置: pruned rows stop at the gate, only kept rows
 *  go up; [aiwillknow] figure 1(a)(b): kept tokens keep their original positions).
 *
 *   dst[r, :width] = src[row_idx[r], :width]       (row_idx NULL: src[r])
 * then, if rope_pos is not NULL, columns [rope_col_begin, rope_col_end) -- whole
 * heads of head_dim columns -- are rotated rotate-half style at position rope_pos[r]:
 *   y[i] = x[i] c - x[i + d/2] s,  y[i + d/2] = x[i + d/2] c + x[i] s,
 *   (c, s) = cos_sin[rope_pos[r]][i], i < d/2 (table from tg_rope_table).
 * src, dst: bf16, row strides ld_src, ld_dst (multiples of 8); width multiple of 8.
 * src has src_rows rows; an index outside [0, src_rows) skips that output row and sets
 * TG_STATUS_BOUNDS (status may be NULL).  dst may equal src (in place) only when
 * row_idx is NULL.  rope_pos values must lie in [0, max_pos); rows outside are copied
 * unrotated and set TG_STATUS_BOUNDS.  Without rope, row_ssq_out (float32, row stride
 * ld_ssq_out >= width / 128, width a multiple of 128; may be NULL) receives the sums of
 * squares of each copied row per 128-column group, for a later folded RMSNorm.
 */
int tg_gather_rope(const tg_bf16* src, int64_t ld_src, int64_t src_rows,
                   const int32_t* row_idx, int64_t n_rows, int width,
                   const int32_t* rope_pos, int rope_col_begin, int rope_col_end,
                   int head_dim, const float* cos_sin, int max_pos, tg_bf16* dst,
                   int64_t ld_dst, float* row_ssq_out, int64_t ld_ssq_out, uint32_t* status,
                   tg_stream_t stream);

/* ------------------------------------------------------------------ KV cache */

/*
 * Compacted KV cache write ([farwalk] How does TokenGate learned token pruning work?:
 * the pruned forward never creates KV entries for pruned tokens; [digest] 方法关键点:
 * the KV cache can be selectively trimmed).
 *   cache_k[slot_offset + r, :width] = k[row_idx[r], :width]   (row_idx NULL: k[r])
 *   cache_v[slot_offset + r, :width] = v[row_idx[r], :width]
 * With row_idx NULL this stores the kept rows' post-RoPE K/V into their cache slots;
 * with row_idx = kept_idx it trims a full-length lower-layer cache to the kept rows.
 * k, v have src_rows rows (indices outside skip the row and set TG_STATUS_BOUNDS);
 * the caches have cache_rows rows and slot_offset + n_rows must not exceed it.
 * All bf16; strides ld_k, ld_v, ld_cache are multiples of 8; width multiple of 8.
 */
int tg_kv_compact(const tg_bf16* k, int64_t ld_k, const tg_bf16* v, int64_t ld_v,
                  int64_t src_rows, const int32_t* row_idx, int64_t n_rows, int width,
                  tg_bf16* cache_k, tg_bf16* cache_v, int64_t ld_cache, int64_t cache_rows,
                  int64_t slot_offset, uint32_t* status, tg_stream_t stream);

/* ------------------------------------------------------------------ attention */

/*
 * Token-gated causal GQA attention over the kept rows
 * ([fluxbbs] 端到端训练的关键在 token 门控注意力: per-head gain on the importance score
 *  added to the logits, SSMax-style temperature from the log-ratio of kept count to
 *  original position; [farwalk] What is token-gated attention?: the score is a bias
 *  on the attention logits; [aiwillknow] figure 1(c): key bias, positive per-head gain).
 * For q head h (kv head g = h / (n_q_heads / n_kv_heads)), request b, query rank r and
 * key rank c <= r (ranks inside the request):
 *   logit = tau_r * (q_r . k_c) / sqrt(head_dim) + gamma[h] * kept_bias[c]
 *   tau_r = beta * ln(r + 1) / ln(p_r + 1),  tau_r = beta when p_r = 0,  p_r = kept_pos[r]
 *   o_r   = sum_c softmax_c(logit) v_c
 * q: bf16 [K_tot, n_q_heads * head_dim] (row stride ld_q); k, v: bf16
 * [K_tot, n_kv_heads * head_dim] (ld_k, ld_v); o: bf16 [K_tot, n_q_heads * head_dim]
 * (ld_o).  lse: float32 [n_q_heads, K_tot] natural-log log-sum-exp, or NULL.
 * kept_pos int32 [K_tot]; kept_bias float32 [K_tot]; gamma float32 [n_q_heads]; beta
 * finite and >= 0 (a temperature scale; otherwise TG_ERR_INVALID_ARGUMENT).
 * The kernel adds the bias term inside the Q K^T MMA (an extra K=16 step whose columns
 * hold gamma_h log2(e) / t_r and kept_bias, each split into two bf16 parts, t_r the
 * row's log2-domain temperature factor), so logits keep fp32 accuracy.
 * Implemented for head_dim = 128 and an even group size n_q_heads / n_kv_heads; q, k,
 * v, o 16-byte aligned with strides that are multiples of 8; at most 512 requests per
 * call.  The kernel runs the two q heads of a kv head on tcgen05 tensor cores with S and
 * O accumulators in tensor memory and a TMA-fed K/V ring.  workspace (16-byte aligned,
 * tg_gated_attention_workspace_size bytes) may be NULL.  status may be NULL.
 */
int tg_gated_attention(const tg_bf16* q, int64_t ld_q, const tg_bf16* k, int64_t ld_k,
                       const tg_bf16* v, int64_t ld_v, const int32_t* cu_kept,
                       const int32_t* cu_kept_host, int batch, int n_q_heads,
                       int n_kv_heads, int head_dim, const int32_t* kept_pos,
                       const float* kept_bias, const float* gamma, float beta, tg_bf16* o,
                       int64_t ld_o, float* lse, void* workspace, size_t workspace_bytes,
                       uint32_t* status, tg_stream_t stream);

/*
 * Workspace bytes that let tg_gated_attention split the key range of long causal query
 * tiles over several CTAs (balancing the triangle over all SMs).  Each part writes its
 * partial result (unnormalised O, row max, row sum) there and counts itself in; the
 * part that completes a tile's count merges the parts and writes o.  0 when the layout
 * needs no split.  With a smaller or NULL workspace the call still runs, one CTA per
 * query tile and kv-head pair.  The workspace must be zero-filled before its first use
 * (the counters); every call that completes leaves it that way.  After a call that
 * raised TG_STATUS_TIMEOUT or TG_STATUS_WORKSPACE, zero it again before reusing it.
 * Layout, for n_items work items and G = n_q_heads / 2 head groups (size = n_items *
 * (n_q_heads * 66560 + 8 * G) bytes): the partial results (66560 bytes per item and q
 * head), then int32 arrival counters [n_items][G], then int32 ready flags [n_items][G].
 * A counter found outside [0, parts) sets TG_STATUS_WORKSPACE; that tile's parts then
 * neither publish nor merge, so its output rows are left unwritten (and a part that
 * already counted itself last waits for a flag that never comes, up to the bounded
 * wait, and sets TG_STATUS_TIMEOUT).
 */
size_t tg_gated_attention_workspace_size(const int32_t* cu_kept_host, int batch,
                                         int n_q_heads, int n_kv_heads, int head_dim);

/*
 * Backward of tg_gated_attention with respect to the gate, what training it end to end
 * needs ([fluxbbs] 端到端训练的关键在 token 门控注意力; [digest] 方法关键点).  Given the
 * forward's inputs, its output o and natural-log lse, and dO = dL/do:
 *   dl[r, c]   = P[r, c] (dO_r . v_c - dO_r . o_r)        (c <= r, same request)
 *   d_bias[c]  = sum_h gamma_h sum_r dl[r, c]              float32 [K_tot], required
 *   d_gamma[h] = sum_{r,c} dl[r, c] kept_bias[c]           float32 [n_q_heads], or NULL
 *   d_beta     = sum_{h,r,c} dl[r, c] (tau_r / beta) q_r.k_c / sqrt(head_dim)   float32 [1], or NULL
 * with P recomputed from q, k, the bias and lse exactly as the forward formed the logits.
 * d_bias is the gradient for kept_bias; the gradient of a prunable token's gate score z is
 * d_bias of its kept row (a question token has none).  Layouts, shapes and limits as
 * tg_gated_attention, and n_q_heads <= 64; d_o: bf16 [K_tot, n_q_heads * head_dim] (ld_do); lse: float32
 * [n_q_heads, K_tot] from that forward call.  workspace: at least
 * tg_gated_attention_bias_grad_workspace_size(...) bytes (no zero-fill needed; 16-byte
 * aligned).  tcgen05 kernel, one CTA per (request, 128-key tile, chunk of query tiles,
 * kv head): S^T = K Q^T (+ the bias step) and dP^T = V dO^T in TMEM, one thread per key;
 * partial sums reduced by two small kernels in a fixed order, so the results are
 * deterministic.  Bounded waits as the forward (TG_STATUS_TIMEOUT).  status may be NULL.
 */
int tg_gated_attention_bias_grad(const tg_bf16* q, int64_t ld_q, const tg_bf16* k,
                                 int64_t ld_k, const tg_bf16* v, int64_t ld_v, const tg_bf16* o,
                                 int64_t ld_o, const tg_bf16* d_o, int64_t ld_do,
                                 const float* lse, const int32_t* cu_kept,
                                 const int32_t* cu_kept_host, int batch, int n_q_heads,
                                 int n_kv_heads, int head_dim, const int32_t* kept_pos,
                                 const float* kept_bias, const float* gamma, float beta,
                                 float* d_bias, float* d_gamma, float* d_beta, void* workspace,
                                 size_t workspace_bytes, uint32_t* status, tg_stream_t stream);
size_t tg_gated_attention_bias_grad_workspace_size(const int32_t* cu_kept_host, int batch,
                                                   int n_q_heads, int n_kv_heads,
                                                   int head_dim);

/*
 * Backward of the gate's scorer: its parameter gradients from dL/d(kept_bias), the
 * gradient tg_gated_attention_bias_grad returns ([fluxbbs] 端到端训练的关键在 token 门控注意力:
 * the gate is trained end to end through the gated attention; [fluxbbs] 门控到底插在模型的
 * 哪个位置: the scorer and the sequence RMSNorm it differentiates).  The top-K choice is
 * piecewise constant and passes no gradient.  With r_t = 1/sqrt(mean(h_t^2) + eps_norm),
 * u_t = W1 (r_t h_t * norm_w), z_t = s_t / rms_b over request b:
 *   dz_t   = d_kept_bias[r] where t = kept_idx[r] is prunable, else 0
 *   ds_t   = (dz_t - z_t m_b) / rms_b,  m_b = mean over the request of dz z
 *   dw2_f  = sum_t ds_t SiLU(u_tf)
 *   dW1[f, i]  = norm_w_i sum_t ds_t w2_f SiLU'(u_tf) r_t h_ti
 *   dnorm_w_i  = sum_f W1[f, i] sum_t ds_t w2_f SiLU'(u_tf) r_t h_ti
 * h, ld_h, total_tokens, hidden, norm_w (NULL = ones), W1, width, w2, eps_norm,
 * cu_seqlens(_host), batch, eps_seq, prunable: as tg_gate_score (hidden a multiple of
 * 128, width 256).  s: float32 [total_tokens], the s_out of tg_gate_score on the same
 * inputs.  cu_kept / cu_kept_host: int32 [batch+1] (K_b <= N_b); kept_idx: int32
 * [K_tot] distinct rows of their request, as tg_topk_compact writes them;
 * d_kept_bias: float32 [K_tot].  Outputs (float32, overwritten): ds_out [total_tokens],
 * dW1 [width, hidden] (row stride hidden), dw2 [width], dnorm_w [hidden] (may be NULL).
 * workspace: tg_gate_score_backward_workspace_size(...) bytes, 16-byte aligned, no
 * zero-fill needed.  The scorer GEMM runs again on tcgen05 with a gradient epilogue
 * (bf16 r_t du_t); the weight gradient h^T (r du) runs on tcgen05 with both operands
 * MN-major, split over tokens; every reduction has a fixed order (bit-reproducible).
 * A kept index outside its request sets TG_STATUS_BOUNDS and is skipped; bounded waits
 * set TG_STATUS_TIMEOUT.  total_tokens = 0 writes zero gradients.  status may be NULL.
 */
int tg_gate_score_backward(const tg_bf16* h, int64_t ld_h, int64_t total_tokens, int hidden,
                           const float* norm_w, const tg_bf16* W1, int width, const float* w2,
                           float eps_norm, const float* s, const int32_t* cu_seqlens,
                           const int32_t* cu_seqlens_host, int batch, float eps_seq,
                           const uint8_t* prunable, const int32_t* cu_kept,
                           const int32_t* cu_kept_host, const int32_t* kept_idx,
                           const float* d_kept_bias, float* ds_out, float* dW1,
                           float* dnorm_w, float* dw2, void* workspace,
                           size_t workspace_bytes, uint32_t* status, tg_stream_t stream);
size_t tg_gate_score_backward_workspace_size(int64_t total_tokens, int hidden, int width,
                                             int batch);

/* ------------------------------------------------------------------ projections */

/*
 * Dense projection used by the gated layers on the kept rows (Wq/Wk/Wv/Wo):
 *   c[m, n] = r_m * sum_k a[m, k] w[n, k]  (+ residual[m, n])
 * with r_m = 1/sqrt(mean_k a[m,k]^2 + eps) when rmsnorm_a is 1 (a pre-attention
 * RMSNorm of weight 1 folded into the epilogue), else r_m = 1.
 * a: bf16 [M, K] (lda); w: bf16 [N, K] (ldw, output rows); c, residual: bf16 [M, N]
 * (ldc, ld_res; residual may be NULL and may equal c).  K multiple of 64, N multiple
 * of 128, strides multiples of 8.  row_ssq_out (may be NULL): float32 [M, N/128] (row
 * stride ld_ssq_out) receiving the sums of squares of each stored bf16 output row per
 * 128 columns (what a following folded RMSNorm needs).  tcgen05 GEMM, TMA-fed, fp32
 * accumulation in TMEM; without rmsnorm_a and with N a multiple of 256 it runs on CTA
 * pairs (tcgen05 cta_group::2, 256 x 256 tiles).  status may be NULL.
 */
int tg_linear(const tg_bf16* a, int64_t lda, const tg_bf16* w, int64_t ldw, tg_bf16* c,
              int64_t ldc, int64_t M, int N, int K, int rmsnorm_a, float eps,
              const tg_bf16* residual, int64_t ld_res, float* row_ssq_out,
              int64_t ld_ssq_out, void* workspace, size_t workspace_bytes, uint32_t* status,
              tg_stream_t stream);

/*
 * Workspace bytes that let the CTA-pair GEMM behind tg_linear, tg_qkv_rope_cache and
 * tg_qkv_qknorm_rope_cache share its last round of 256 x 256 tiles along K over all
 * clusters (stream-K tail): when the tiles leave that round partly idle, every cluster
 * takes an equal run of the remaining k-blocks; the piece holding a tile's first k-block
 * adds the others' fp32 partial sums in k order before its epilogue (so the result is
 * deterministic; it differs from the unsplit call only by fp32 summation order), and the
 * launch is cooperative.  Those calls take (workspace, workspace_bytes): NULL or fewer
 * bytes runs unsplit.  Zero-fill the workspace once before its first use (its ready
 * flags); every completed call leaves it so; calls whose GPU work can overlap must not
 * share one.  The size depends only on the device (its number of SM pairs: partial sums
 * of 256 KB per cluster plus the flags).  Not part of the method: a scheduling device.
 */
size_t tg_gemm_workspace_size(void);

/*
 * One gated layer's QKV projection with RoPE and the compacted KV-cache write fused into
 * the GEMM epilogue ([aiwillknow] figure 1(a)(b): kept tokens keep their original
 * positions, upper layers store KV only for kept tokens; [farwalk] How does TokenGate
 * learned token pruning work?):
 *   a = RMSNorm(x) (weight 1, eps);  [Q | K | V] = a w_qkv^T;
 *   q_out[r]                = RoPE(Q[r], pos[r])
 *   cache_k[slot_offset+r]  = RoPE(K[r], pos[r]);  cache_v[slot_offset+r] = V[r]
 * RoPE is rotate-half on every head with the table of tg_rope_table, applied to the fp32
 * accumulators before the single rounding to bf16.  Equivalent to tg_linear (rmsnorm=1)
 * followed by tg_gather_rope (rope mode) and tg_kv_compact, in one kernel.
 * x: bf16 [M, hidden] (ld_x); w_qkv: bf16 [(n_q_heads + 2 n_kv_heads) * head_dim, hidden]
 * (rows: Wq, Wk, Wv); pos: int32 [M] (values < max_pos, else TG_STATUS_BOUNDS and the
 * row uses position 0), or NULL: then cos_sin is the per-row table of tg_rope_rows for
 * these M rows and max_pos its row stride ld_rot (>= M, else TG_ERR_INVALID_ARGUMENT);
 * q_out: bf16 [M, n_q_heads * head_dim] (ld_q); cache_k/cache_v:
 * bf16 rows of n_kv_heads * head_dim (ld_cache).  head_dim = 128, hidden multiple of 64.
 * row_ssq_in (may be NULL): float32 [M, hidden/128] (row stride ld_ssq_in) holding the
 * sums of squares of x per 128 columns (from tg_gather_rope or tg_linear row_ssq_out);
 * with it the norm needs no extra read of x and the GEMM runs on CTA pairs; without it
 * the norm is accumulated from x inside the GEMM.  status may be NULL.
 */
int tg_qkv_rope_cache(const tg_bf16* x, int64_t ld_x, const tg_bf16* w_qkv, int64_t ld_w,
                      int64_t M, int hidden, int n_q_heads, int n_kv_heads, int head_dim,
                      float eps, const int32_t* pos, const float* cos_sin, int max_pos,
                      tg_bf16* q_out, int64_t ld_q, tg_bf16* cache_k, tg_bf16* cache_v,
                      int64_t ld_cache, int64_t slot_offset, const float* row_ssq_in,
                      int64_t ld_ssq_in, void* workspace, size_t workspace_bytes,
                      uint32_t* status, tg_stream_t stream);

/*
 * tg_qkv_rope_cache with QK-norm, for a full (Qwen3-shaped) layer body: each Q and K
 * head of a row is RMS-normalised over its head_dim values and multiplied by q_norm_w
 * or k_norm_w (float32 [head_dim], shared by the heads) before RoPE:
 *   Q_h <- Q_h / sqrt(mean(Q_h^2) + eps) * q_norm_w  (K likewise with k_norm_w)
 * in fp32 from the accumulators, then RoPE and the single rounding to bf16.  The layer
 * body comes from the page [fluxbbs] (门控到底插在模型的哪个位置) evaluating a Qwen3 model;
 * the QK-norm itself is that model's, not the pages'.  Requires row_ssq_in and Q/K/V
 * widths that are multiples of 256 (CTA-pair kernel): else TG_ERR_INVALID_ARGUMENT /
 * TG_ERR_UNSUPPORTED_SHAPE.  A weighted pre-attention RMSNorm is folded into w_qkv
 * beforehand with tg_fold_norm_weight.  Other arguments as tg_qkv_rope_cache.
 */
int tg_qkv_qknorm_rope_cache(const tg_bf16* x, int64_t ld_x, const tg_bf16* w_qkv,
                             int64_t ld_w, int64_t M, int hidden, int n_q_heads, int n_kv_heads,
                             int head_dim, float eps, const float* q_norm_w,
                             const float* k_norm_w, const int32_t* pos, const float* cos_sin,
                             int max_pos, tg_bf16* q_out, int64_t ld_q, tg_bf16* cache_k,
                             tg_bf16* cache_v, int64_t ld_cache, int64_t slot_offset,
                             const float* row_ssq_in, int64_t ld_ssq_in, void* workspace,
                             size_t workspace_bytes, uint32_t* status, tg_stream_t stream);

/*
 * Up half of the SwiGLU MLP of a full layer body (pruned tokens skip the upper MLPs as
 * well: [fluxbbs] 门控到底插在模型的哪个位置):
 *   b = RMSNorm(x) (eps; the norm weight folded into w_gu by tg_pack_gate_up),
 *   h_out[m, f] = SiLU(b . W_gate[f]) * (b . W_up[f]),  SiLU(v) = v / (1 + e^-v)
 * evaluated in fp32 from the two accumulators, one rounding to bf16.
 * x: bf16 [M, hidden] (ld_x); row_ssq_in: float32 [M, hidden/128] (ld_ssq_in, required:
 * the row sums of squares tg_linear's row_ssq_out gives); w_gu: bf16 [2 ffn, hidden]
 * (ld_w) in the layout tg_pack_gate_up writes; h_out: bf16 [M, ffn] (ld_h).  hidden and
 * ffn multiples of 128, strides multiples of 8, 16-byte aligned bases.  CTA-pair
 * tcgen05 GEMM over 256 x 256 tiles of the interleaved weight.  The down projection is
 * tg_linear(h_out, W_down, x, residual = x).  status may be NULL.
 */
int tg_swiglu(const tg_bf16* x, int64_t ld_x, const tg_bf16* w_gu, int64_t ld_w, int64_t M,
              int hidden, int ffn, float eps, const float* row_ssq_in, int64_t ld_ssq_in,
              tg_bf16* h_out, int64_t ld_h, uint32_t* status, tg_stream_t stream);

/*
 * Weight preparation, once per model load (not per step).
 * tg_fold_norm_weight: out[r, c] = bf16(w[r, c] * norm_w[c]) for an RMSNorm weight that
 *   multiplies the input of w (w: bf16 [rows, cols], ld_w; out may equal w).
 * tg_pack_gate_up: out = bf16 [2 ffn, hidden] with rows 128 j .. 128 j + 63 = W_gate rows
 *   64 j .. 64 j + 63 and rows 128 j + 64 .. 128 j + 127 = the same W_up rows, every
 *   column c multiplied by norm_w[c] (norm_w may be NULL: no scaling).  ffn multiple of
 *   64.  w_gate, w_up: bf16 [ffn, hidden] (ld_gate, ld_up); out must not alias them.
 * Both are asynchronous on `stream`.
 */
int tg_fold_norm_weight(const tg_bf16* w, int64_t ld_w, int64_t rows, int cols,
                        const float* norm_w, tg_bf16* out, int64_t ld_out, tg_stream_t stream);
int tg_pack_gate_up(const tg_bf16* w_gate, int64_t ld_gate, const tg_bf16* w_up, int64_t ld_up,
                    int ffn, int hidden, const float* norm_w, tg_bf16* out, int64_t ld_out,
                    tg_stream_t stream);

/*
 * One layer boundary in one launch: the output projection of gated layer l followed by
 * gated layer l+1's QKV projection, RoPE and KV-cache write, with identical results to
 *   tg_linear(o, W_o, x, residual = x, row_ssq)            (x <- x + o W_o^T)
 *   tg_qkv_rope_cache(x, W_qkv, ..., row_ssq_in = row_ssq)
 * Both run on the CTA-pair kernel over 256 x 256 tiles: the projection's tiles first,
 * then the QKV tiles, each of which starts once every projection tile of its 256 rows
 * has stored them (counted in `workspace`), so the QKV work fills the SMs the projection
 * leaves idle instead of waiting for a second launch.
 * o: bf16 [M, o_cols] (ld_o); w_o: bf16 [hidden, o_cols] (ld_wo); x: bf16 [M, hidden]
 * (ld_x, updated in place); row_ssq: float32 [M, hidden/128] (ld_ssq) receives the new
 * rows' sums of squares per 128 columns and feeds the folded RMSNorm of the QKV part;
 * the remaining arguments are those of tg_qkv_rope_cache.  hidden, n_q_heads*head_dim
 * and n_kv_heads*head_dim must be multiples of 256; head_dim 128; o_cols multiple of 64.
 * workspace: tg_out_proj_qkv_workspace_size(M) bytes, 4-byte aligned, zero-filled before
 * its first use; every completed call leaves it zeroed (after TG_STATUS_TIMEOUT, zero it
 * again).  The launch is cooperative (all its CTAs resident at once); a device that
 * cannot hold them returns TG_ERR_CUDA.
 */
int tg_out_proj_qkv_next(const tg_bf16* o, int64_t ld_o, const tg_bf16* w_o, int64_t ld_wo,
                         tg_bf16* x, int64_t ld_x, float* row_ssq, int64_t ld_ssq, int64_t M,
                         int hidden, int o_cols, const tg_bf16* w_qkv, int64_t ld_wqkv,
                         int n_q_heads, int n_kv_heads, int head_dim, float eps,
                         const int32_t* pos, const float* cos_sin, int max_pos, tg_bf16* q_out,
                         int64_t ld_q, tg_bf16* cache_k, tg_bf16* cache_v, int64_t ld_cache,
                         int64_t slot_offset, void* workspace, size_t workspace_bytes,
                         uint32_t* status, tg_stream_t stream);

/* Workspace bytes of tg_out_proj_qkv_next for M rows (two int32 counters per 256 rows). */
size_t tg_out_proj_qkv_workspace_size(int64_t M);

#ifdef __cplusplus
}
#endif

#endif /* TOKENGATE_H */
