/*
 * gmla.h — C ABI of the Gated Multi-head Latent Attention hot path (B200, sm_100a).
 *
 * What is computed (sources cited by page title and section):
 *
 *   "Gated MLA 计算公式：输出门与 FFN 的区别" (hackcha.cn)
 *     §一   c_s = W_c x_s;  k_s^(h) = W_k^(h) c_s;  v_s^(h) = W_v^(h) c_s
 *     §二   a_{t,s} = Softmax_{s<=t}(q_t^(h) . k_s^(h) / sqrt(d_h)),  o_t^(h) = sum_s a_{t,s} v_s^(h)
 *           õ_t = Concat_h o_t^(h);   y_t = W_o [ Sigmoid(W_g x_t) ⊙ õ_t ]   (boxed equation)
 *     §四   NoPE: no positional encoding on q and k.
 *   "Gated Multi-head Latent Attention (Gated MLA)" (codewithdark-git.github.io)
 *     "Gating Mechanism": per-head gate g_h = sigmoid(W_g x + b_g) scaling head h.
 *   "LLM 注意力与计算内核精读笔记 · 03 注意力头变体：MQA / GQA / MLA" (zzszmyf.github.io)
 *     §5.1  only c_s is cached; W_k and W_v are absorbed at inference time.
 *     §5.2  decoupled RoPE: k^R_s = RoPE(W_kr x_s) is cached beside c_s, shared by
 *           all heads; q^R gets its own rotated d_R dims per head.
 *     §5.3  a cached row holds d_c + d_R elements (576 for d_c=512, d_R=64).
 *     题4   absorption identity q^T W_k c = (W_k^T q)^T c.
 *
 * Readings where the pages leave a step open (shared with the oracle):
 *   q^(h) = W_q^(h) x (full-rank query, no bias); softmax_scale is passed in
 *   (1/sqrt(d_h), or 1/sqrt(d_h + d_R) with the decoupled RoPE key); RoPE rotates
 *   pairs (2i, 2i+1) by pos * base^(-2i/d_R); a decode query is at position
 *   seq_len - 1 and attends to all seq_len cached rows.
 *
 * Conventions for every entry point:
 *   - Every pointer argument is a DEVICE pointer owned by the caller unless its
 *     comment says otherwise; the library keeps none of them after the call.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream). The returned status covers argument checks and the
 *     launches. Faults seen by a kernel (a device wait that timed out, a
 *     sequence longer than its cache) are written to a status word at the start
 *     of `workspace` and returned by gmla_sync_status().
 *   - Row-major layouts. Weights are [out, in]:
 *       W_c [d_c, d_model]   W_kr [d_R, d_model]    W_q [H*d_h, d_model]
 *       W_qr [H*d_R, d_model]  W_k, W_v [H, d_h, d_c]
 *       with a compressed query (d_cq > 0): W_dq [d_cq, d_model], W_uq [H*d_h, d_cq],
 *       W_qr [H*d_R, d_cq], and W_q unused
 *       W_g [G, d_model] with G = H*d_h (per-channel gate) or G = H (per-head gate)
 *       b_g [G] (fp32, optional)   W_o [d_model, H*d_h]
 *     Weights, x, q, the cache, o and y use the config's dtype (bf16 or fp32);
 *     gate logits and b_g are always fp32; index arrays are int32.
 *   - The bf16 path runs on tcgen05 tensor cores with fp32 accumulation; the
 *     fp32 path runs on CUDA cores in fp32. There is no CPU fallback: a shape
 *     the kernels do not cover returns GMLA_ERR_UNSUPPORTED.
 *   - All base pointers must be 16-byte aligned.
 */
#ifndef GMLA_H_
#define GMLA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GMLA_API __attribute__((visibility("default")))
#else
#define GMLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum gmla_status {
  GMLA_OK = 0,
  GMLA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, inconsistent sizes */
  GMLA_ERR_UNSUPPORTED = 2,   /* valid but not covered by the kernels (no fallback) */
  GMLA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than the *_workspace_size query */
  GMLA_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed; see gmla_last_error() */
  GMLA_ERR_TIMEOUT = 5,       /* a device-side wait gave up (reported by gmla_sync_status) */
  GMLA_ERR_DEVICE_RANGE = 6   /* a kernel saw an out-of-range length/page (gmla_sync_status) */
} gmla_status;

typedef enum gmla_dtype { GMLA_BF16 = 0, GMLA_FP32 = 1 } gmla_dtype;

/* Latent cache element format. GMLA_CACHE_SAME: the config's dtype.
 * GMLA_CACHE_FP8_E4M3: one byte per element, an E4M3 code (round to nearest
 * even, saturating at +-448) of value / cache_scale, one fp32 scale for the
 * whole cache. It halves the cache bytes a decode reads; the "Kimi K3" gating
 * blog (zwxr.cn) §7 warns that quantisation errors compound, and the library
 * keeps every other operand near bf16 precision. bf16 dtype only: decode
 * (NoPE, d_c = 512) reads it and gmla_latent_project writes it; gmla_prefill
 * over an FP8 cache returns GMLA_ERR_UNSUPPORTED. */
typedef enum gmla_cache_dtype { GMLA_CACHE_SAME = 0, GMLA_CACHE_FP8_E4M3 = 1 } gmla_cache_dtype;

/* Per-channel gate: G = H*d_h ("Gated MLA 计算公式" §二 boxed equation).
 * Per-head gate:    G = H, broadcast over the head's d_h channels
 *                   ("Gated Multi-head Latent Attention", "Gating Mechanism").
 * Per-head hard and quantised gates ("Gated Multi-head Latent Attention",
 * "Variants / Extensions": Hard Gating, Quantized Gates), also G = H:
 *   GMLA_GATE_HEAD_TOPK     1 for the gate_topk heads with the largest logits of
 *                           the token (equal logits: lower head first), else 0
 *   GMLA_GATE_HEAD_BINARY   1 where sigmoid(z) >= 1/2 (z >= 0), else 0
 *   GMLA_GATE_HEAD_TERNARY  sigmoid(z) rounded to the nearest of 0, 1/2, 1
 *                           (halves up): 0 below z = -ln 3, 1 from z = ln 3
 * A head whose gate is 0 contributes exactly 0, so gmla_decode skips its
 * attention (its absorbed query rows are left out of the score products). */
typedef enum gmla_gate_mode {
  GMLA_GATE_CHANNEL = 0,
  GMLA_GATE_HEAD = 1,
  GMLA_GATE_HEAD_TOPK = 2,
  GMLA_GATE_HEAD_BINARY = 3,
  GMLA_GATE_HEAD_TERNARY = 4
} gmla_gate_mode;

typedef struct gmla_config {
  int32_t d_model;
  int32_t n_heads;        /* H */
  int32_t d_h;            /* head dim of q, k, v */
  int32_t d_c;            /* latent dim (cached) */
  int32_t d_rope;         /* decoupled RoPE dims d_R; 0 = NoPE */
  int32_t gate_mode;      /* gmla_gate_mode */
  int32_t gate_bias;      /* 1: b_g is given */
  float softmax_scale;    /* scale applied to q.k (+ q^R.k^R) before the softmax */
  float rope_base;        /* RoPE base (e.g. 10000) */
  int32_t dtype;          /* gmla_dtype */
  int32_t d_cq;           /* low-rank query width d_cq ("精读笔记 03" §5.1: c^Q = W^DQ h,
                             q = W^UQ c^Q; §5.2: q^R = RoPE(W^QR c^Q)); 0 = full-rank query */
  int32_t gate_topk;      /* k of GMLA_GATE_HEAD_TOPK (1 <= k <= H); ignored otherwise */
  int32_t cache_dtype;    /* gmla_cache_dtype: the latent cache's element format */
  float cache_scale;      /* GMLA_CACHE_FP8_E4M3: a stored code e means cache_scale * e */
} gmla_config;

typedef struct gmla_weights {
  const void* W_c;
  const void* W_kr;       /* NULL when d_rope == 0 */
  const void* W_q;
  const void* W_qr;       /* NULL when d_rope == 0 */
  const void* W_k;
  const void* W_v;
  const void* W_g;
  const float* b_g;       /* NULL unless gate_bias */
  const void* W_o;
  const void* W_dq;       /* [d_cq, d_model] when d_cq > 0, else NULL */
  const void* W_uq;       /* [H*d_h, d_cq] when d_cq > 0, else NULL */
} gmla_weights;

/* Latent cache. A row holds [c (d_c) | k^R (d_R)] of one token, d_c + d_R
 * elements ("精读笔记 03" §5.2). Nothing gate-related is cached: the gate
 * depends only on the current token ("Gated MLA 计算公式" §五).
 *   contiguous (paged = 0): data = [batch, capacity, d_c + d_R]
 *   paged      (paged = 1): data = [num_pages, page_size, d_c + d_R];
 *     token p of sequence b lives in page block_table[b*max_pages_per_seq + p/page_size]
 *     at row p % page_size. block_table is a device int32 array. */
typedef struct gmla_cache {
  void* data;
  int32_t paged;
  int32_t batch;              /* contiguous: sequences held */
  int32_t capacity;           /* contiguous: rows per sequence */
  int32_t page_size;          /* paged: rows per page (multiple of 8) */
  int32_t num_pages;          /* paged: pages in the pool */
  int32_t max_pages_per_seq;  /* paged: row length of block_table */
  const int32_t* block_table; /* paged: [batch, max_pages_per_seq] */
} gmla_cache;

/* ---------------------------------------------------------------------------
 * gmla_latent_project — everything computed from the tokens' own hidden states.
 *   x            [T, d_model]
 *   positions    [T] int32, position of each token within its sequence
 *   seq_ids      [T] int32, sequence (cache slot) of each token
 *   cache        receives row [c | RoPE(W_kr x, pos)] of every token at (seq_id, position)
 *                ("Gated MLA 计算公式" §一; "精读笔记 03" §5.1, §5.2)
 *   q_out        [T, H, d_h + d_R]: q^(h) = W_q^(h) x, then q^R = RoPE(W_qr^(h) x, pos);
 *                with d_cq > 0: c^Q = W_dq x, q = W_uq c^Q, q^R = RoPE(W_qr c^Q, pos)
 *                ("精读笔记 03" §5.1, §5.2), two GEMMs with c^Q kept in the workspace
 *   gate_logits  [T, G] fp32: W_g x (+ b_g)
 *   workspace    device scratch of gmla_latent_project_workspace_size(cfg, T) bytes
 * Rows of the cache not addressed by (seq_id, position) are left untouched.
 * Returns GMLA_ERR_INVALID_ARG if T < 0 or a pointer is missing/misaligned.
 * ------------------------------------------------------------------------- */
GMLA_API gmla_status gmla_latent_project(const gmla_config* cfg, const gmla_weights* w,
                                const void* x, int32_t T,
                                const int32_t* positions, const int32_t* seq_ids,
                                const gmla_cache* cache,
                                void* q_out, float* gate_logits,
                                void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * gmla_decode — one query token per sequence against its cached rows, in the
 * absorbed form ("精读笔记 03" §5.1, 题4): scores are (W_k^T q) . c_s (+ q^R . k^R_s),
 * the weighted sum is taken over latents and W_v is applied afterwards; the
 * sigmoid gate is applied before the result leaves the chip.
 *   q            [B, H, d_h + d_R] (as written by gmla_latent_project)
 *   gate_logits  [B, G] fp32, or NULL to write the ungated head outputs
 *   seq_lens     [B] int32: cached rows of each sequence INCLUDING the query's
 *                own row; the query sits at position seq_len - 1. A length of 0
 *                yields o = 0; a length beyond the cache sets
 *                GMLA_ERR_DEVICE_RANGE in the status word and yields o = 0.
 *   o_gated      [B, H*d_h] = gate ⊙ Concat_h o^(h)
 *   workspace    device scratch of gmla_decode_workspace_size(cfg, B) bytes
 * ------------------------------------------------------------------------- */
GMLA_API gmla_status gmla_decode(const gmla_config* cfg, const gmla_weights* w,
                        const void* q, const float* gate_logits,
                        const gmla_cache* cache, const int32_t* seq_lens, int32_t B,
                        void* o_gated, void* workspace, size_t workspace_bytes,
                        void* stream);

/* ---------------------------------------------------------------------------
 * gmla_prefill — causal attention of whole prompts in the explicit form
 * ("Gated MLA 计算公式" §一, §二): K^(h) = C W_k^(h)T and V^(h) = C W_v^(h)T are
 * rebuilt from the cached latents, then softmax_{s<=t}(q_t . k_s * scale) V,
 * gated on the way out.
 *   q            [T, H, d_h + d_R], packed by sequence
 *   gate_logits  [T, G] fp32, or NULL for ungated output
 *   cu_seqlens   [B+1] int32 device prefix sums of the prompt lengths
 *                (sequence b occupies packed rows cu_seqlens[b] .. cu_seqlens[b+1]-1
 *                and cache positions 0 .. len-1 of cache slot b)
 *   T, max_seqlen host copies of cu_seqlens[B] and the longest prompt
 *   o_gated      [T, H*d_h]
 *   workspace    device scratch of gmla_prefill_workspace_size(cfg, T, B) bytes
 * ------------------------------------------------------------------------- */
GMLA_API gmla_status gmla_prefill(const gmla_config* cfg, const gmla_weights* w,
                         const void* q, const float* gate_logits,
                         const gmla_cache* cache, const int32_t* cu_seqlens,
                         int32_t B, int32_t T, int32_t max_seqlen,
                         void* o_gated, void* workspace, size_t workspace_bytes,
                         void* stream);

/* ---------------------------------------------------------------------------
 * gmla_gate_out — y = W_o [ sigmoid(gate_logits) ⊙ o ] ("Gated MLA 计算公式" §二).
 *   o            [T, H*d_h]; already gated when gate_logits is NULL
 *   gate_logits  [T, G] fp32 or NULL
 *   y            [T, d_model]
 *   workspace    device scratch of gmla_gate_out_workspace_size(cfg, T) bytes
 * ------------------------------------------------------------------------- */
GMLA_API gmla_status gmla_gate_out(const gmla_config* cfg, const gmla_weights* w,
                          const void* o, int32_t T, const float* gate_logits,
                          void* y, void* workspace, size_t workspace_bytes,
                          void* stream);

/* ---------------------------------------------------------------------------
 * gmla_decode_noalloc — gmla_decode for callers that cannot allocate device
 * memory: engines and plugins whose device memory belongs to their own pool,
 * and loops that cannot pay cudaMalloc's implicit synchronisation. The pages
 * have no counterpart to this call: it is a deployment convenience.
 * Same arguments and results as gmla_decode, minus the workspace: the scratch
 * is a 16 MiB array in the library's device memory, held by every GPU that
 * loads the library until the process exits. The call allocates nothing.
 *   - Batches whose gmla_decode_workspace_size() exceeds 16 MiB are rejected
 *     with GMLA_ERR_WORKSPACE (use gmla_decode with a workspace instead).
 *   - The first call on a device looks up the array's device address.
 *   - All calls share the array and it keeps the previous call's contents:
 *     calls whose kernels overlap on the GPU race on it, so serialise them.
 *   - Device-side faults are recorded in the shared array's status word,
 *     which each call clears first; this variant does not report them back.
 *     A sequence length beyond the cache or a page id outside the pool
 *     therefore gives an undefined o_gated with no error returned: callers
 *     that cannot vouch for seq_lens and the block table should use
 *     gmla_decode, whose workspace status gmla_sync_status() reads.
 *   - An invalid configuration or B < 0 returns GMLA_ERR_INVALID_ARG before
 *     anything reaches the device.
 * ------------------------------------------------------------------------- */
GMLA_API gmla_status gmla_decode_noalloc(const gmla_config* cfg, const gmla_weights* w,
                                         const void* q, const float* gate_logits,
                                         const gmla_cache* cache, const int32_t* seq_lens,
                                         int32_t B, void* o_gated, void* stream);

/* ---------------------------------------------------------------------------
 * Context-parallel decode: one sequence's cache split across R GPUs (ranks),
 * each holding a range of its positions. The softmax over all L rows is the
 * one of "Gated MLA 计算公式" §二; it decomposes over disjoint ranges: a range
 * r gives O_r = sum_{s in r} e^{z_s - M_r} c_s / l_r and the log-sum-exp
 * lse_r = M_r + log l_r, and O_lat = sum_r e^{lse_r - M} O_r / sum_r e^{lse_r - M}
 * with M = max_r lse_r. Each rank calls gmla_decode_partial on its rows, the
 * partials of all ranks are gathered (one NCCL all-gather of
 * R x B x H x (d_c + 4) floats, outside the library), and any rank calls
 * gmla_decode_merge, which applies W_v and the gate as gmla_decode does.
 *
 * gmla_decode_partial — gmla_decode restricted to cached positions
 * [seq_starts[b], seq_ends[b]) of each sequence (bf16 path).
 *   q, gate_logits, cache, B, workspace: as gmla_decode (the workspace size is
 *                gmla_decode_workspace_size(cfg, B)); gate logits only matter
 *                for hard / quantised gates, whose zero-gated heads are skipped
 *   seq_starts   [B] int32 or NULL (= 0): first position this rank attends to;
 *                the rows of the cache below it are never used
 *   seq_ends     [B] int32: one past the last position (<= the cache's rows)
 *   partial      [B, H, d_c + 4] fp32: per (sequence, head) the normalised
 *                latent output O_r (d_c values), then lse_r in log2 units
 *                (-inf for an empty range or a skipped head), then 3 zeros
 * gmla_decode_merge — merges R partials into o_gated.
 *   partials     [R, B, H, d_c + 4] fp32 (the gathered partials, rank-major)
 *   gate_logits  [B, G] fp32 or NULL (ungated), as gmla_decode
 *   o_gated      [B, H*d_h]
 *   workspace    gmla_decode_merge_workspace_size(cfg, B) bytes
 * ------------------------------------------------------------------------- */
GMLA_API gmla_status gmla_decode_partial(const gmla_config* cfg, const gmla_weights* w,
                                         const void* q, const float* gate_logits,
                                         const gmla_cache* cache, const int32_t* seq_starts,
                                         const int32_t* seq_ends, int32_t B, float* partial,
                                         void* workspace, size_t workspace_bytes, void* stream);
GMLA_API gmla_status gmla_decode_merge(const gmla_config* cfg, const gmla_weights* w,
                                       const float* partials, int32_t R, const float* gate_logits,
                                       int32_t B, void* o_gated, void* workspace,
                                       size_t workspace_bytes, void* stream);
GMLA_API size_t gmla_decode_merge_workspace_size(const gmla_config* cfg, int32_t B);

/* Scratch sizes in bytes (0 is never returned; 256-byte aligned). An invalid
 * configuration or a negative size gets 256 (the calls themselves then fail
 * with GMLA_ERR_INVALID_ARG). */
GMLA_API size_t gmla_latent_project_workspace_size(const gmla_config* cfg, int32_t T);
GMLA_API size_t gmla_decode_workspace_size(const gmla_config* cfg, int32_t B);
GMLA_API size_t gmla_prefill_workspace_size(const gmla_config* cfg, int32_t T, int32_t B);
GMLA_API size_t gmla_gate_out_workspace_size(const gmla_config* cfg, int32_t T);

/* Zero the status word of a workspace (stream-ordered). */
GMLA_API gmla_status gmla_clear_status(void* workspace, void* stream);

/* Synchronise `stream`, then return the device status word kept in
 * `workspace` (GMLA_OK, GMLA_ERR_TIMEOUT or GMLA_ERR_DEVICE_RANGE). */
GMLA_API gmla_status gmla_sync_status(const void* workspace, void* stream);

/* Static description of a status code. */
GMLA_API const char* gmla_status_string(gmla_status s);

/* Message of the last failing call on this host thread ("" if none). */
GMLA_API const char* gmla_last_error(void);

/* ---------------------------------------------------------------------------
 * Launch accounting and opt-in per-kernel timing (instrumentation, not part of
 * the method). With profiling enabled, the library records a CUDA event pair
 * on the launching stream around each of its kernel launches; records are
 * kept until the next gmla_profile_enable call.
 * ------------------------------------------------------------------------- */
/* Kernels launched by this process so far (all devices, all streams). */
GMLA_API uint64_t gmla_launch_count(void);
/* Enable (1) or disable (0) per-launch timing; both clear the records. */
GMLA_API gmla_status gmla_profile_enable(int32_t enable);
/* Number of recorded launches. */
GMLA_API int32_t gmla_profile_count(void);
/* Name and duration (ms) of record i; waits for its stop event. */
GMLA_API gmla_status gmla_profile_get(int32_t i, const char** name, float* ms);

/* ---------------------------------------------------------------------------
 * Test hook, not part of the method: arms (1) or disarms (0) a one-shot stall
 * in the next bf16 gmla_decode on this process. In that call the tensor-core
 * thread of the first attention block waits on a barrier that nothing
 * completes; the wait gives up after its bound (about one second), the block
 * leaves through its abort path, the workspace status word reads
 * GMLA_ERR_TIMEOUT and the call's output is undefined. The device stays
 * usable: clear the status and call again. Faults nothing, hangs nothing.
 * ------------------------------------------------------------------------- */
GMLA_API gmla_status gmla_test_stall_next_decode(int32_t enable);

/* Library version, e.g. "gmla 0.1.0 sm_100a". */
GMLA_API const char* gmla_version(void);

#ifdef __cplusplus
}
#endif
#endif /* GMLA_H_ */
