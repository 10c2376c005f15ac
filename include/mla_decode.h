/*
 * mla_decode.h — C ABI of the B200 (sm_100a) MLA absorbed-decode library.
 *
 * The operation is the decode step of DeepSeek-V2's Multi-head Latent Attention with
 * weight absorption. Sources, by page title and section:
 *   [V2-walk]  "DeepSeek-V2 paper walkthrough" (2kiu.com/news/6085339): §2.3 matrix
 *              absorption (displayed equation), §2.4 decoupled RoPE.
 *   [V2-arch]  "Transformer-15: DeepSeek-V2 architecture" (zeeklog.com): MHA equations,
 *              eqs. 9-11 (c^KV, k^C = W^UK c^KV, v^C = W^UV c^KV), cache table.
 *   [V2-notes] "DeepSeek-V2" paper notes (process-cxr.github.io): shared k^R, cache of
 *              d_c + d_h^R values per token.
 *   [V3-walk]  "DeepSeek-V3 technical report walkthrough" (2kiu.com/news/6340724):
 *              §2.2 only c^KV and k^R are cached, §2.3 absorption and RoPE.
 *
 * Shapes: n_h heads (1..128), d_h = 128, d_c = 512, d_R = d_h^R = 64; one cache row is
 * [c^KV (512) ; k^R (64)] = 576 bf16 values, one copy for all heads. bf16 means IEEE
 * bfloat16; every bf16 output is rounded to nearest-even from fp32.
 *
 * Conventions for every call:
 *   - Memory: the caller owns every input and output buffer; all of them are DEVICE
 *     pointers on the handle's device unless stated. The handle owns only its workspace
 *     (split partials, work list, device error word), allocated in mla_decode_create;
 *     the compute calls never allocate.
 *   - Asynchrony: every compute call enqueues kernels on `stream` and returns at once.
 *     The returned status covers argument checks and launch errors only. A device-side
 *     problem (a page-table entry out of range, a bounded wait that ran out) sets the
 *     handle's device error word; read it with mla_check_device_errors.
 *   - Threads: a handle may be used by one stream at a time (its workspace is shared by
 *     the calls enqueued on it).
 *   - Alignment: every pointer must be 16-byte aligned.
 *   - Status codes are the MLA_* values below; mla_status_string names them.
 */
#ifndef MLA_DECODE_H
#define MLA_DECODE_H

#include <stdint.h>

/* Only the functions below are exported from libmla_decode.so (it is built with hidden
 * visibility for everything else). */
#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct mla_decode_s* mla_handle_t;
typedef struct CUstream_st* mla_stream_t; /* same object as cudaStream_t; NULL = legacy default stream */

enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = -1,  /* a pointer, size or layout argument is invalid          */
  MLA_ERR_UNSUPPORTED = -2,  /* valid, but outside what this build implements           */
  MLA_ERR_CUDA = -3,         /* a CUDA runtime/driver call failed (launch, alloc, ...)  */
  MLA_ERR_OOM = -4,          /* workspace allocation failed in mla_decode_create        */
  MLA_ERR_DEVICE_CHECK = -5  /* the device error word was set (bad page id, timeout)    */
};

typedef struct {
  int32_t n_heads;       /* n_h, 1..128                                               */
  int32_t d_head;        /* d_h, must be 128                                          */
  int32_t d_latent;      /* d_c, must be 512                                          */
  int32_t d_rope;        /* d_h^R, must be 64                                         */
  int32_t page_size;     /* 0 = contiguous cache; else tokens per page, must be 64    */
  int32_t max_batch;     /* largest batch any call will pass (>= 1)                   */
  int64_t max_kv_len;    /* largest kv_len any call will pass (>= 1)                  */
  float softmax_scale;   /* 0 => 1/sqrt(d_h + d_h^R) = 1/sqrt(192)                    */
  float rope_base;       /* RoPE base (10000 for DeepSeek-V2); 0 => q^R not rotated   */
  int32_t max_splits;    /* upper bound on KV splits per sequence; 0 => automatic     */
  /* YaRN context extension of the decoupled RoPE ([V2-arch] pre-training paragraph;
   * [V2-notes] Long-Context Extension: s = 40, alpha = 1, beta = 32 over a 4K original
   * context, sqrt(t) = 0.0707 ln s + 1). With yarn_factor s > 1, pair m's frequency
   * theta_m = base^(-2m/64) becomes (1 - g) theta_m / s + g theta_m, where
   * g = clamp((r - alpha) / (beta - alpha), 0, 1) and r = original_len * theta_m / (2 pi)
   * (the YaRN method's blend), for the rotated query (mla_absorb_q) and the written key
   * (mla_append_kv); and softmax_scale 0 then means t / sqrt(192), t = (coef ln s + 1)^2.
   * yarn_factor 0 or 1 leaves RoPE and the scale as above. */
  float yarn_factor;        /* s: 0 or 1 => off, else >= 1                              */
  int32_t yarn_original_len;/* original context length (>= 1 when on; 4096)             */
  float yarn_alpha;         /* ramp start, in wavelengths per original context (1)      */
  float yarn_beta;          /* ramp end, > yarn_alpha (32)                               */
  float yarn_mscale_coef;   /* coefficient of ln s in sqrt(t), >= 0 (0.0707)            */
  /* New tokens per sequence per call, T (multi-token prediction / speculative decoding:
   * [V3-walk] §4.1, the MTP modules' extra tokens verified by the main model). 0 or 1 =>
   * one. With T > 1 every per-sequence array below gains a token axis after the batch axis
   * (q_c [batch, T, n_h, 128], q_abs [batch, T, n_h, 576], out_latent [batch, T, n_h, 512],
   * lse [batch, T, n_h], latent/out of mla_apply_wuv, hidden [batch, T, d] of
   * mla_append_kv); kv_lens counts the T new tokens, which sit at positions kv_len - T + t;
   * token t attends to rows 0 .. kv_len - T + t (a token with none: latent 0, lse -inf) and
   * its q^R is rotated at max(kv_len - T + t, 0). Limits: n_heads * T <= 2^20 and
   * max_batch * T <= 8192 (the cache write's workspace holds max_batch * T rows of 2.3 KB
   * each); mla_decode_attn runs more than 128 attention rows per sequence in groups of 128,
   * each reading the cache, which suits a few draft tokens; a long prompt (prefill) goes
   * through mla_prefill_attn. */
  int32_t q_len;
} mla_config_t;

/*
 * Check a configuration without touching any GPU: MLA_OK if mla_decode_create would accept
 * it, else the status it would return (MLA_ERR_INVALID_ARG / MLA_ERR_UNSUPPORTED).
 */
MLA_API int mla_check_config(const mla_config_t* cfg);

/*
 * Create a handle on CUDA device `device` and allocate its workspace there (sized from
 * cfg->max_batch, cfg->max_kv_len and n_heads). On success *out is the handle and the
 * return is MLA_OK; on failure *out is NULL. Makes `device` current on the calling thread.
 */
MLA_API int mla_decode_create(const mla_config_t* cfg, int device, mla_handle_t* out);

/* Free the workspace and the handle. Synchronises the device first. NULL is a no-op. */
MLA_API int mla_destroy(mla_handle_t h);

/*
 * Query absorption and RoPE ([V2-walk] §2.3 displayed equation: q^T W_UK c = (W_UK^T q)^T c;
 * [V3-walk] §2.3; [V2-walk] §2.4 decoupled query):
 *   q_abs[b,i,0:512]   = W_UK,i^T q^C_{b,i}                     (fp32 accumulation)
 *   q_abs[b,i,512:576] = RoPE_{kv_lens[b]-1}(q^R_{b,i})         (pairs (2m,2m+1),
 *                        angle (kv_len-1) * base^(-2m/64); identity if rope_base == 0)
 * q_c   bf16 [batch, n_h, 128]  the content query (W^UQ c^Q, computed upstream)
 * q_r   bf16 [batch, n_h, 64]   the decoupled query, not yet rotated
 * w_uk  bf16 [n_h, 128, 512]    W_UK,i maps a latent (512) to head i's content key (128);
 *                               this is the nn.Linear weight [n_h*128, 512] reshaped
 * kv_lens int32 [batch]         cached tokens per sequence (the new token included); the
 *                               query sits at position kv_lens[b]-1 (0 if kv_lens[b] == 0)
 * q_abs bf16 [batch, n_h, 576]  output
 * Errors: MLA_ERR_INVALID_ARG for NULL pointers or batch outside 1..max_batch.
 */
MLA_API int mla_absorb_q(mla_handle_t h, int32_t batch, const void* q_c, const void* q_r,
                 const void* w_uk, const int32_t* kv_lens, void* q_abs, mla_stream_t stream);

/*
 * Split-KV decode attention over the shared latent cache ([V2-walk] §2.3: the weighted
 * sum stays in the latent space; [V2-notes] shared k^R; [V3-walk] §2.2 cached rows):
 *   s_{b,i,j}  = scale * q_abs[b,i,:] . [c^KV_j ; k^R_j]          j = 0 .. kv_lens[b]-1
 *   out_latent[b,i,:] = sum_j softmax_j(s)_j c^KV_j                (512, bf16)
 *   lse[b,i]   = log sum_j exp(s_{b,i,j})                         (natural log, fp32)
 * q_abs  bf16 [batch, n_h, 576] (from mla_absorb_q)
 * c_kv   bf16 cache rows, row r at c_kv + r*row_stride (512 values each)
 * k_r    bf16 cache rows, row r at k_r + r*row_stride (64 values each); the usual fused
 *        layout is k_r = c_kv + 512 with row_stride = 576
 * row_stride  elements between consecutive rows; a multiple of 8, >= 512
 * seq_stride  contiguous cache (page_size 0): token j of sequence b is row b*seq_stride+j,
 *             seq_stride >= max kv_len; ignored for a paged cache
 * kv_lens int32 [batch], each 0..max_kv_len. kv_len 0 gives latent 0 and lse = -inf.
 * page_table  paged cache only (else NULL): int32 [batch, max_pages]; token j of sequence b
 *             is row page_table[b*max_pages + j/page_size]*page_size + j%page_size. Only the
 *             first ceil(kv_len/page_size) entries of a row are read. An entry outside
 *             0..num_pages-1 sets the device error word; its tokens are skipped.
 * max_pages, num_pages  table width and physical pages in the pool (paged only)
 * out_latent bf16 [batch, n_h, 512]  output
 * lse   fp32 [batch, n_h] output, or NULL to skip
 * Errors: MLA_ERR_INVALID_ARG for NULL pointers, bad strides or alignment, a page table
 * given to a contiguous handle (or missing for a paged one), max_pages too small for
 * max_kv_len.
 */
MLA_API int mla_decode_attn(mla_handle_t h, int32_t batch, const void* q_abs, const void* c_kv,
                    const void* k_r, int64_t row_stride, int64_t seq_stride,
                    const int32_t* kv_lens, const int32_t* page_table, int32_t max_pages,
                    int32_t num_pages, void* out_latent, float* lse, mla_stream_t stream);

/*
 * Prefill: the attention of a prompt's T = q_len new tokens over the latent cache, the same
 * results as mla_decode_attn with this handle (token t of sequence b attends to cache rows
 * 0 .. kv_len[b] - T + t, the causal mask of [V2-arch]'s MHA equations, softmax over j = 1..t)
 * for long prompts ([V2-notes] "Inference cost": prompt input throughput is a headline figure
 * of the deployed model). One kernel: each work item is one head and 128 consecutive new tokens
 * of one sequence (128 attention rows sharing every cache row they read), taken whole by one
 * 2-CTA cluster over the rows its last token sees, with the normalised latent written directly
 * (no split partials, no merge).
 *   q_abs      bf16 [batch, T, n_h, 576] (mla_absorb_q with this handle)
 *   cache      as for mla_decode_attn (bf16 only)
 *   out_latent bf16 [batch, T, n_h, 512]; lse fp32 [batch, T, n_h] or NULL
 * A token that sees no row gets latent 0 and lse -inf. Errors as for mla_decode_attn.
 */
MLA_API int mla_prefill_attn(mla_handle_t h, int32_t batch, const void* q_abs, const void* c_kv,
                     const void* k_r, int64_t row_stride, int64_t seq_stride,
                     const int32_t* kv_lens, const int32_t* page_table, int32_t max_pages,
                     int32_t num_pages, void* out_latent, float* lse, mla_stream_t stream);

/*
 * mla_decode_attn over a quantised cache ([V2-notes] Inference cost: the deployed KV cache is
 * quantised, to about 6 bits per element on average; the format is this library's reading):
 * cached row r is 576 OCP FP8 E4M3 codes [c^KV (512) ; k^R (64)] at kv_codes + r*row_stride
 * (bytes) and one power-of-two scale 2^kv_exp[r]; its values are 2^kv_exp[r] times the codes'
 * values. Row r is indexed as for mla_decode_attn (b*seq_stride + j, or the page table). The
 * scores, softmax and latent sum are those of mla_decode_attn on the dequantised rows (which
 * are exact in bf16). kv_exp int8, one per row; row_stride a multiple of 16, >= 576. Outputs,
 * kv_lens, page table and errors as for mla_decode_attn.
 */
MLA_API int mla_decode_attn_fp8(mla_handle_t h, int32_t batch, const void* q_abs, const void* kv_codes,
                        const int8_t* kv_exp, int64_t row_stride, int64_t seq_stride,
                        const int32_t* kv_lens, const int32_t* page_table, int32_t max_pages,
                        int32_t num_pages, void* out_latent, float* lse, mla_stream_t stream);

/*
 * mla_decode_attn over one shard of each sequence's cache, for a request whose tokens are
 * spread over several GPUs: the same attention over the rows this caller holds (kv_lens =
 * the rows held, 0 allowed), with out_latent as fp32 [batch, (T,) n_h, 512] (normalised over
 * the shard) and lse required. q_abs must be rotated at the request's global position
 * (mla_absorb_q with the global kv_lens): the cached k^R rows carry their global positions.
 * The shards' results are merged with mla_merge_partials. Not on the pages: the split-KV
 * log-sum-exp merge across GPUs is this library's. MLA_ERR_UNSUPPORTED with q_len > 1 (the
 * causal limits of several new tokens follow their global positions).
 */
MLA_API int mla_decode_attn_partial(mla_handle_t h, int32_t batch, const void* q_abs, const void* c_kv,
                            const void* k_r, int64_t row_stride, int64_t seq_stride,
                            const int32_t* kv_lens, const int32_t* page_table, int32_t max_pages,
                            int32_t num_pages, float* out_latent, float* lse, mla_stream_t stream);

/*
 * Log-sum-exp merge of n_parts partial results over disjoint pieces of each sequence's cache:
 *   lse* = max_p lse_p, w_p = exp(lse_p - lse*),
 *   out_latent = sum_p w_p latent_p / sum_p w_p (bf16), lse = lse* + log sum_p w_p (fp32).
 * latent_parts fp32 [n_parts][batch][(T,) n_h][512], lse_parts fp32 [n_parts][batch][(T,) n_h]
 * (the outputs of mla_decode_attn_partial stacked part by part, e.g. by an all-gather across
 * GPUs); out_latent bf16 [batch, (T,) n_h, 512]; lse fp32 or NULL. Parts are added in part
 * order, so the result does not depend on timing. A row whose parts are all empty (lse -inf)
 * gets latent 0 and lse -inf.
 * Errors: MLA_ERR_INVALID_ARG for NULL pointers, batch outside 1..max_batch, n_parts < 1,
 * misalignment.
 */
MLA_API int mla_merge_partials(mla_handle_t h, int32_t batch, int32_t n_parts, const float* latent_parts,
                       const float* lse_parts, void* out_latent, float* lse, mla_stream_t stream);

/*
 * V up-projection ([V2-walk] §2.3: W_UV is applied last; [V2-arch] eq. 11 v^C = W^UV c^KV):
 *   out[b,i,:] = W_UV,i latent[b,i,:]                               (fp32 accumulation)
 * latent bf16 [batch, n_h, 512]; w_uv bf16 [n_h, 128, 512]; out bf16 [batch, n_h, 128].
 */
MLA_API int mla_apply_wuv(mla_handle_t h, int32_t batch, const void* latent, const void* w_uv,
                  void* out, mla_stream_t stream);

/*
 * One whole decode step ([V2-walk] §2.3, the absorbed inference path): mla_absorb_q, then
 * mla_decode_attn, then mla_apply_wuv, with the same arguments and the same results, in one
 * call. The split-KV work plan, which mla_decode_attn builds in a launch of its own, is built
 * here by one extra block of the absorption kernel, beside the heads.
 *   q_abs  bf16 [batch, (q_len,) n_h, 576] and latent bf16 [batch, (q_len,) n_h, 512]: device
 *          scratch for the intermediate results, 16-byte aligned, left holding them;
 *   out    bf16 [batch, (q_len,) n_h, 128].
 * Every argument is checked before anything is launched (MLA_ERR_INVALID_ARG, nothing queued).
 * Device errors (a kv_len outside 0..max_kv_len, a page-table entry out of range) are
 * reported as for the three calls.
 */
MLA_API int mla_decode_step(mla_handle_t h, int32_t batch, const void* q_c, const void* q_r,
                    const void* w_uk, const void* w_uv, const void* c_kv, const void* k_r,
                    int64_t row_stride, int64_t seq_stride, const int32_t* kv_lens,
                    const int32_t* page_table, int32_t max_pages, int32_t num_pages, void* q_abs,
                    void* latent, void* out, mla_stream_t stream);

/*
 * FP8 weights for the two head projections ([V3-walk] section 4.4: weights quantised in
 * 1 x 128 tiles with high-precision accumulation; section 5.5: FP8 for storage with the
 * arithmetic in BF16 is the safe first step; [V2-notes] "Inference cost": the deployed model
 * converts its parameters to FP8). A weight W [n_h * 128, 512] (W_UK or W_UV as nn.Linear
 * weights, the [n_h, 128, 512] arrays above) is given as
 *   w_codes  uint8 [n_h * 128, 512]: E4M3 codes (OCP FP8 E4M3: bias 7, no infinities, code
 *            0x7F/0xFF NaN), 16-byte aligned;
 *   w_exp    int8  [n_h * 128, 4]:   one exponent e per 1 x 128 tile, the tile of row r
 *            covering latent columns [128 t, 128 t + 128); e in -126..127;
 * and stands for W[r, c] = value(w_codes[r, c]) * 2^w_exp[r, c / 128]. Each such value is a
 * bf16 number, so the results are those of mla_absorb_q / mla_apply_wuv on the dequantised
 * weights (the same products, accumulated in fp32). Other arguments and errors as there.
 */
MLA_API int mla_absorb_q_fp8(mla_handle_t h, int32_t batch, const void* q_c, const void* q_r,
                     const void* w_uk_codes, const int8_t* w_uk_exp, const int32_t* kv_lens,
                     void* q_abs, mla_stream_t stream);

MLA_API int mla_apply_wuv_fp8(mla_handle_t h, int32_t batch, const void* latent, const void* w_uv_codes,
                      const int8_t* w_uv_exp, void* out, mla_stream_t stream);

/*
 * Cache write of the step's new token ([V2-arch] eq. 9 c^KV = W^DKV h; [V2-notes]
 * architecture: an RMSNorm follows the compressed latent; [V3-walk] §2.2 k^R = RoPE(W^KR h)
 * and only c^KV and k^R are cached):
 *   x          = [W_DKV ; W_KR] hidden[b,:]                         (576, fp32 accumulation)
 *   c^KV row   = x[0:512] / sqrt(mean(x[0:512]^2) + rms_eps) * gamma      (bf16)
 *   k^R  row   = RoPE_{kv_lens[b]-1}(x[512:576])                          (bf16; pairs
 *                (2m,2m+1), angle (kv_len-1) * base^(-2m/64); identity if rope_base == 0)
 * written as token kv_lens[b]-1 of sequence b, in the layout mla_decode_attn reads; no other
 * row is touched.
 * d_model     hidden size d: a multiple of 64, 64..8192 (5120 for DeepSeek-V2)
 * hidden      bf16 [batch, d_model]  the token's hidden state h_t (after the block's input norm)
 * w_dkv       bf16 [512, d_model]    W^DKV, the nn.Linear weight of the down-projection
 * w_kr        bf16 [64, d_model]     W^KR
 * gamma       bf16 [512]             the latent RMSNorm's weight
 * rms_eps     >= 0 and finite (1e-6 in DeepSeek-V2)
 * c_kv, k_r, row_stride, seq_stride, page_table, max_pages, num_pages: the cache, as for
 *             mla_decode_attn, here written
 * kv_lens     int32 [batch], each 1..max_kv_len: tokens of the sequence with the new one;
 *             a value outside that range (there is no row to write) or a page-table entry
 *             outside 0..num_pages-1 sets the device error word and the sequence is skipped
 * Errors: MLA_ERR_INVALID_ARG for NULL pointers, batch outside 1..max_batch, d_model not a
 * positive multiple of 64, a bad rms_eps, strides or alignment, a page table given to a
 * contiguous handle (or missing for a paged one); MLA_ERR_UNSUPPORTED for d_model > 8192.
 */
MLA_API int mla_append_kv(mla_handle_t h, int32_t batch, int32_t d_model, const void* hidden,
                  const void* w_dkv, const void* w_kr, const void* gamma, float rms_eps,
                  void* c_kv, void* k_r, int64_t row_stride, int64_t seq_stride,
                  const int32_t* kv_lens, const int32_t* page_table, int32_t max_pages,
                  int32_t num_pages, mla_stream_t stream);

/*
 * mla_append_kv into a quantised cache (the layout of mla_decode_attn_fp8): the new row's 576
 * values, computed as above in fp32, get the smallest power-of-two scale 2^e with
 * max|row| / 2^e <= 448 (e in -126..127, 0 for an all-zero row), and each value / 2^e is
 * rounded to the nearest E4M3 code, ties to even (saturating at +-448). Codes go to
 * kv_codes + r*row_stride (bytes; a multiple of 16, >= 576), e to kv_exp[r]. Other arguments
 * and errors as for mla_append_kv.
 */
MLA_API int mla_append_kv_fp8(mla_handle_t h, int32_t batch, int32_t d_model, const void* hidden,
                      const void* w_dkv, const void* w_kr, const void* gamma, float rms_eps,
                      void* kv_codes, int8_t* kv_exp, int64_t row_stride, int64_t seq_stride,
                      const int32_t* kv_lens, const int32_t* page_table, int32_t max_pages,
                      int32_t num_pages, mla_stream_t stream);

/*
 * mla_decode_attn for callers that cannot allocate device memory. The pages have no
 * counterpart to this call: it exists for library users whose device memory is owned by
 * someone else (a serving engine that has reserved nearly all of HBM for its own KV-cache
 * pool and allocates only from it, a plugin host whose memory manager forbids cudaMalloc)
 * or whose hot path cannot afford cudaMalloc/cudaFree and the synchronisation they may
 * bring. Such callers cannot create a handle, so the configuration comes as arguments and
 * the scratch (work plan, split partials, error word) lives in one fixed 32 MiB array of
 * device memory inside the library, which every GPU that loads the library holds until the
 * process exits. The call allocates nothing.
 *
 * Arguments and results are those of mla_decode_attn, with n_heads, softmax_scale (0 =>
 * 1/sqrt(192)), page_size (0 or 64) and max_kv_len in place of the handle, and:
 *   err_word  device uint32, or NULL: set to 0 at the start of the call, then OR-ed with the
 *             device error bits of mla_check_device_errors; with NULL the bits stay in the
 *             library's array and are not reported.
 * Uses the current device. Limits: batch <= 64 and n_heads <= 128; beyond them the call
 * returns MLA_ERR_UNSUPPORTED and enqueues nothing. The split count adapts to what fits in
 * the array, so results can differ from mla_decode_attn by floating-point reassociation.
 * All calls on a device share the array and it keeps the last call's contents: calls whose
 * kernels overlap on the GPU (different streams or host threads) race, so serialise them.
 * The first call on a device looks up the array's device address; make it before any
 * stream capture. A look-up that fails returns MLA_ERR_CUDA and is retried by the next call.
 */
MLA_API int mla_decode_attn_noalloc(int32_t n_heads, float softmax_scale, int32_t page_size,
                            int64_t max_kv_len, int32_t batch, const void* q_abs,
                            const void* c_kv, const void* k_r, int64_t row_stride,
                            int64_t seq_stride, const int32_t* kv_lens,
                            const int32_t* page_table, int32_t max_pages, int32_t num_pages,
                            void* out_latent, float* lse, uint32_t* err_word,
                            mla_stream_t stream);

/*
 * Synchronise `stream`, then read and clear the handle's device error word. Returns MLA_OK
 * if it was clear, MLA_ERR_DEVICE_CHECK if a kernel set it (*detail, if not NULL, gets the
 * word: bit 0 = page-table entry out of range, bit 1 = a bounded wait ran out, bit 2 = a
 * kv_len outside 0..max_kv_len, clamped, or outside 1..max_kv_len in mla_append_kv), or
 * MLA_ERR_CUDA if the synchronisation itself failed.
 */
MLA_API int mla_check_device_errors(mla_handle_t h, mla_stream_t stream, uint32_t* detail);

/* Bytes of device workspace the handle holds. */
MLA_API int64_t mla_workspace_bytes(mla_handle_t h);

/* A static, human-readable name for a status code. */
MLA_API const char* mla_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* MLA_DECODE_H */
