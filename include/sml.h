/*
 * sml.h -- C ABI of libsml.so, the sparse-MLA decode step of a DeepSeek-style
 * sparse attention layer (Mistral Large 4 as served by vLLM) on one NVIDIA
 * B200 (sm_100a):
 *
 *   sml_indexer_scores     DSA indexer: FP8 q.k per indexer head, ReLU,
 *                          head-weighted sum, over a paged FP8 indexer cache
 *   sml_topk               exact per-query top-k over those scores
 *   sml_sparse_mla_decode  absorbed-query MLA over only the selected tokens of
 *                          a paged fp8_ds_mla latent cache (split over the
 *                          selected keys, then a log-sum-exp merge)
 *   sml_run_layer          the three in a row, or only the attention for a
 *                          shared-indexer layer that reuses a prior top-k
 *   sml_indexer_k_cache_write, sml_latent_cache_write, sml_indexer_q_quant
 *                          the producers just before the step: FP8
 *                          quantisation of new tokens into the two caches,
 *                          and of the indexer queries
 *   sml_dcp_pack_candidates, sml_dcp_merge_candidates,
 *   sml_dcp_split_selection, sml_lse_combine
 *                          decode context parallelism: the steps between the
 *                          ranks' own top-k and sparse MLA
 *
 * Sources: vLLM blog "vLLM 首日支持 Mistral Large 4：1T 参数 MoE 多模态模型",
 * highlights list (MLA with KV LoRA rank 512 and RoPE dim 64; a DSA indexer
 * picks the top 2048 keys per query; default fp8_ds_mla latent cache) and
 * section "实现细节 / 模型架构" (sparse MLA over the fp8_ds_mla latent cache plus
 * an indexer over an FP8 indexer cache; shared-indexer layers reuse the top-k
 * of the preceding indexer layer; the indexer has its own SSMax; NoPE layers
 * are MLA with RoPE dim 0 over the same kernels and cache layout; 47,136 B of
 * KV per token).  The pages print no formula, layout or API; where they are
 * silent this header states the reading it implements.
 *
 * Conventions for every entry point
 *   - All array pointers are DEVICE pointers on the current CUDA device unless
 *     a comment says "host".  The caller owns every buffer; the library
 *     allocates nothing and frees nothing.
 *   - Work is enqueued on `stream` (a cudaStream_t, NULL = legacy default
 *     stream) and returns without waiting.  Only sml_read_device_status
 *     synchronises (that stream).
 *   - Return value: SML_OK, or a negative SML_ERR_* code.  On an error nothing
 *     has been enqueued, and sml_last_error() (per host thread) lists every
 *     check that failed, not only the first.
 *   - Checks that need device data (context lengths, block-table entries,
 *     selected indices) run inside the kernels: a bad value sets a bit in a
 *     sticky status word in the workspace and the access is skipped (masked);
 *     kernels never trap.  Read it with sml_read_device_status.
 *   - Supported shapes (anything else returns SML_ERR_UNSUPPORTED): page size
 *     64 tokens; num_heads in {16, 32, 64, 128}; 1 <= topk <= 2048;
 *     rope_dim in {0, 64}; 64 indexer heads of dim 128.
 *
 * Notation: B requests; T query tokens in total; request r owns query tokens
 * [cu_q[r], cu_q[r+1]) (Q_r = cu_q[r+1] - cu_q[r] >= 1) and L_r = ctx_len[r]
 * cached tokens, its own query tokens included (L_r >= Q_r).  Query j (0-based)
 * of request r sees positions [0, n_t) with n_t = L_r - Q_r + j + 1 (causal
 * within the request), unless sml_problem.vis_len gives n_t.  Logical
 * position s of request r lives in physical page
 * block_table[r * max_pages + s / 64], row s % 64.
 */
#ifndef SML_H_
#define SML_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes --------------------------------------------------------- */
#define SML_OK 0
#define SML_ERR_INVALID_ARG (-1)  /* a NULL pointer, negative size, inconsistent sizes */
#define SML_ERR_UNSUPPORTED (-2)  /* a shape or option outside the supported set */
#define SML_ERR_WORKSPACE (-3)    /* workspace NULL, misaligned or smaller than sml_workspace_size */
#define SML_ERR_CUDA (-4)         /* a CUDA runtime call failed (launch, attribute) */
#define SML_ERR_DEVICE_FAULT (-5) /* returned by sml_read_device_status: a device check failed */
#define SML_ERR_TIMEOUT (-6)      /* returned by sml_read_device_status: a bounded wait gave up */

/* Bits of the device status word (see sml_read_device_status). */
#define SML_FAULT_PAGE 0x1        /* a block-table entry outside [0, num_pages) */
#define SML_FAULT_INDEX 0x2       /* a selected position outside [0, n_t) */
#define SML_FAULT_LENGTHS 0x4     /* cu_q / ctx_len inconsistent with the problem */
#define SML_FAULT_TOPK_LEN 0x8    /* a top-k length outside [0, min(topk, n_t)] */
#define SML_FAULT_TIMEOUT 0x10    /* an mbarrier or flag wait exceeded its poll limit */

/* ---- fixed sizes (readings of the pages' byte counts) --------------------- */
#define SML_PAGE_TOKENS 64
#define SML_LATENT_DIM 512          /* KV LoRA rank */
#define SML_ROPE_DIM 64
/* fp8_ds_mla row, 656 B: [512 x e4m3 latent][4 x fp32 scale, one per 128
 * elements][64 x bf16 RoPE key]; a page is 64 rows back to back. */
#define SML_LATENT_ROW_BYTES 656
#define SML_LATENT_PAGE_BYTES (SML_PAGE_TOKENS * SML_LATENT_ROW_BYTES)
/* indexer page: [64 x 128 B e4m3 keys][64 x fp32 per-token scale], 132 B/token */
#define SML_INDEX_HEADS 64
#define SML_INDEX_DIM 128
#define SML_INDEX_PAGE_BYTES (SML_PAGE_TOKENS * (SML_INDEX_DIM + 4))
#define SML_MAX_TOPK 2048

/* Workspace stages for sml_workspace_size. */
#define SML_STAGE_INDEXER 1
#define SML_STAGE_TOPK 2
#define SML_STAGE_MLA 3
#define SML_STAGE_LAYER 4

/* One batch of query tokens.  Host struct; the pointers in it are device
 * pointers.  Every entry point validates it. */
typedef struct sml_problem {
  int32_t num_requests;        /* B >= 1 */
  int32_t num_tokens;          /* T = cu_q[B] >= 1 */
  int32_t num_heads;           /* H, MLA query heads: 16, 32, 64 or 128 */
  int32_t topk;                /* K, 1..2048 */
  int32_t rope_dim;            /* 64 (RoPE layer) or 0 (NoPE layer) */
  int32_t max_pages;           /* row stride of block_table, >= ceil(L_r / 64) */
  int32_t max_ctx;             /* >= every L_r; row stride of the score matrix */
  int32_t ssmax;               /* 0 = off; 1 = scale logits by s * ln(n_t) */
  float sm_scale;              /* softmax scale sigma of the MLA logits */
  float ssmax_s;               /* SSMax s of the MLA logits */
  float ssmax_s_index;         /* SSMax s of the indexer scores */
  const int32_t* cu_q;         /* [B + 1], cu_q[0] = 0, non-decreasing */
  const int32_t* ctx_len;      /* [B], L_r */
  const int32_t* block_table;  /* [B * max_pages], physical page ids */
  /* Optional per-token overrides (NULL = the causal rule; a zero-initialised
   * struct keeps it).  vis_len [T]: n_t itself, in [0, L_r] and
   * non-decreasing within a request (n_t = 0: nothing visible; with it the
   * only length rule on L_r is 0 <= L_r <= max_ctx).  ssmax_len [T]: the n of
   * every SSMax factor s * ln(n), >= 1 (default n_t).  Decode context
   * parallelism sets both: a rank sees its own share of each query's
   * context, but every rank scales by the global length. */
  const int32_t* vis_len;
  const int32_t* ssmax_len;
} sml_problem;

/* Latent cache formats (sml_cache.format of a latent pool; an indexer pool
 * takes 0).  SML_LATENT_E4M3 is the plain per-tensor E4M3 cache of the blog's
 * section "ROCm 实现细节", paragraph "FP8 潜在缓存": all 576 latent dims in FP8
 * under one per-tensor scale, 576 B per token.  Reading: a row is
 * [512 x e4m3 latent][64 x e4m3 RoPE key], value = code * scale.
 * SML_LATENT_BF16 is the unquantised cache the same paragraph compares with,
 * 1,152 B per token: a row is [512 x bf16 latent][64 x bf16 RoPE key],
 * little-endian (sml_cache.scale is ignored).  Sparse MLA over it runs bf16 x
 * bf16 products with fp32 accumulation and bf16 weights split in two terms
 * (16 significant bits); its 128-key tile fills one shared-memory buffer, so
 * its row copies do not overlap the tile's products as the E4M3 formats' do. */
#define SML_LATENT_FP8_DS_MLA 0
#define SML_LATENT_E4M3 1
#define SML_LATENT_E4M3_ROW_BYTES 576
#define SML_LATENT_E4M3_PAGE_BYTES (SML_PAGE_TOKENS * SML_LATENT_E4M3_ROW_BYTES)
#define SML_LATENT_BF16 2
#define SML_LATENT_BF16_ROW_BYTES 1152
#define SML_LATENT_BF16_PAGE_BYTES (SML_PAGE_TOKENS * SML_LATENT_BF16_ROW_BYTES)

/* A paged cache pool: num_pages pages starting at base (256-B aligned).  A
 * zero-initialised descriptor (format 0) is the fp8_ds_mla latent layout or
 * the indexer layout. */
typedef struct sml_cache {
  const void* base;
  int64_t num_pages;
  int32_t format;   /* latent pools: SML_LATENT_*; indexer pools: 0 */
  float scale;      /* SML_LATENT_E4M3: the pool's scale, finite and > 0; else ignored */
} sml_cache;

/* Bytes of workspace the given stage needs for this problem (0 on invalid
 * arguments; see sml_last_error).  SML_STAGE_LAYER covers sml_run_layer,
 * including the score matrix it keeps internally.  A workspace must be
 * 256-B aligned and initialised once with sml_workspace_init; after that it may
 * be reused by any later call whose size fits, on the same stream. */
size_t sml_workspace_size(const sml_problem* p, int stage);

/* Zero the workspace header (device status word and the per-row arrival
 * counters of the two-level top-k).  Call once after allocating a workspace. */
int sml_workspace_init(void* workspace, size_t ws_bytes, void* stream);

/* DSA indexer scores.
 *   I[t, s] = c_t * sq_t * sk_s * sum_h w[t, h] * ReLU(sum_d e4m3(q8[t,h,d]) * e4m3(k8[s,d]))
 * for s < n_t, with c_t = ssmax_s_index * ln(n_t) when ssmax, else 1.
 * (Reading: the pages print no formula for the indexer; this is the
 * DeepSeek-style indexer -- an FP8 dot product per indexer head, a ReLU and a
 * weighted sum over heads -- with head weights per query token and head; both
 * FP8 scales are positive, so they commute with the ReLU.)
 *   iq8       [T, 64, 128] e4m3 codes of the indexer query
 *   iq_scale  [T] fp32 per-token query scale sq_t (> 0)
 *   iw        [T, 64] fp32 head weights
 *   index_cache  pool of SML_INDEX_PAGE_BYTES pages
 *   scores    [T, max_ctx] fp32 out; entries s >= n_t are not written
 * FP8 products are exact; sums accumulate in fp32. */
int sml_indexer_scores(const sml_problem* p, const void* iq8, const float* iq_scale, const float* iw,
                       sml_cache index_cache, float* scores, void* workspace, size_t ws_bytes,
                       void* stream);

/* Exact top-k per query token over scores[t, 0:n_t) (blog section "ROCm
 * 实现细节", persistent decode paragraph: the selection is an exact
 * top-2048).  Order: larger score first; -0.0 == +0.0; a NaN ranks below every
 * number; equal scores go to the lower position.
 *   scores   [T, max_ctx] fp32 (row stride max_ctx), read for s < n_t only
 *   idx      [T, topk] int32 out: the selected positions in ASCENDING order,
 *            then -1 padding
 *   idx_len  [T] int32 out: min(topk, n_t)
 * cu_q / ctx_len inconsistent with the problem set SML_FAULT_LENGTHS (the row
 * gets len 0); a copy of a row's scores into shared memory that outlives its
 * wait limit sets SML_FAULT_TIMEOUT (that row's selection is then unspecified). */
int sml_topk(const sml_problem* p, const float* scores, int32_t* idx, int32_t* idx_len,
             void* workspace, size_t ws_bytes, void* stream);

/* Absorbed-query sparse MLA over the selected positions.  For token t, head h,
 * selected set S_t = idx[t, 0:idx_len[t]):
 *   z_i = sm_scale * c_t * (q[t,h,0:512] . c_hat_i + q[t,h,512:576] . k_pe_i)
 *   out[t,h,:] = sum_i softmax(z)_i * c_hat_i,  lse[t,h] = ln sum_i exp(z_i)
 * with c_hat_i = e4m3 latent * its block scale (SML_LATENT_E4M3: code * the
 * pool scale; SML_LATENT_BF16: the bf16 value), c_t = ssmax_s * ln(n_t) when
 * ssmax, else 1.  rope_dim = 0 (NoPE) drops the k_pe term.
 *   q        [T, H, 512 + rope_dim] bf16
 *   latent   pool of pages of its format's page size
 *   idx      [T, topk] int32 logical positions (any order; -1 padding ignored)
 *   idx_len  [T] int32 number of valid entries at the front of each idx row
 *   out      [T, H, 512] fp32;  lse [T, H] fp32 (natural log; -inf if empty)
 * Arithmetic: both products run on the tensor cores as E4M3 x E4M3 with fp32
 * accumulation, straight from the cached E4M3 codes (the latent is never
 * dequantised).  The bf16 query of each head is split exactly into two E4M3
 * terms, q = s_h (hi + lo), s_h the power of two >= amax_h / 448: exact for
 * every query element at or above 2^-6 s_h, E4M3's smallest normal step (a
 * bf16 has 8 significant bits, hi takes 4, lo the other 4); smaller elements
 * keep an absolute error below 2^-10 s_h (half of E4M3's subnormal step).
 * The RoPE part (fp8_ds_mla) runs as bf16 x bf16.  The softmax is fp32; each
 * weight 2^(z_i - M_h) * block scale is split into three E4M3 terms whose sum
 * carries 12 significant bits, with M_h a per-head integer exponent that keeps
 * every weight at most 440 and the dominant ones at or above 4 (in E4M3's
 * normal range).  A SML_LATENT_BF16 pool runs bf16 x bf16 products instead,
 * with the bf16 query as given and each weight split into two bf16 terms.
 * Ordering: the kernel starts early behind the previous kernel of `stream`
 * and reads the problem's cu_q, ctx_len, vis_len and ssmax_len, and q, before
 * it waits for that kernel (idx, idx_len and the cache after), so those must
 * not be written by the call of this library just before it. */
int sml_sparse_mla_decode(const sml_problem* p, const void* q, sml_cache latent,
                          const int32_t* idx, const int32_t* idx_len, float* out, float* lse,
                          void* workspace, size_t ws_bytes, void* stream);

/* One layer.  If reuse_idx is NULL: indexer scores (kept in the workspace),
 * top-k into idx_out / len_out, then sparse MLA over them.  If reuse_idx is not
 * NULL (a shared-indexer layer): sparse MLA over reuse_idx / reuse_len only;
 * iq8, iq_scale, iw, index_cache, idx_out and len_out may then be NULL. */
int sml_run_layer(const sml_problem* p, const void* q, const void* iq8, const float* iq_scale,
                  const float* iw, sml_cache latent, sml_cache index_cache,
                  const int32_t* reuse_idx, const int32_t* reuse_len, int32_t* idx_out,
                  int32_t* len_out, float* out, float* lse, void* workspace, size_t ws_bytes,
                  void* stream);

/* Sparse MLA decode for callers that cannot allocate device memory: same
 * arguments, checks and results as sml_sparse_mla_decode, but no workspace.
 * (The pages have no counterpart; this is an interface convenience.)
 * Some callers cannot pass a workspace: a serving engine that has handed all
 * spare HBM to its KV-cache pool at start-up, a host runtime that forbids
 * cudaMalloc on its hot path because it synchronises the device, or a plugin
 * with no handle on its host's allocator.  This entry point keeps its split
 * partials in a scratch array built into libsml.so instead: 16 MiB held on
 * every GPU that loads the library, until the process exits.  It allocates and
 * frees nothing.
 *   - A problem whose partials (T x H x splits x 2,052 B) exceed 16 MiB returns
 *     SML_ERR_UNSUPPORTED; use sml_sparse_mla_decode for it.
 *   - The first call on a device looks up the scratch array's device address
 *     (once per device); make that first call before any stream capture.
 *   - Every call on a device shares the one scratch array and it keeps the last
 *     call's contents (nothing in it needs to start at zero).  Calls that can
 *     overlap on the GPU (different streams, or several host threads) race on
 *     it: serialise them.
 *   - There is no workspace, so the device checks (out-of-range pages or
 *     positions, a bounded wait that gave up) set bits in a status word built
 *     into the library beside the scratch array: one per device, shared by
 *     every call on it and sticky until cleared.  Read it with
 *     sml_noalloc_read_status. */
int sml_sparse_mla_decode_noalloc(const sml_problem* p, const void* q, sml_cache latent,
                                  const int32_t* idx, const int32_t* idx_len, float* out, float* lse,
                                  void* stream);

/* The status word of sml_sparse_mla_decode_noalloc on the current device, as
 * sml_read_device_status reads a workspace's: synchronise `stream`, then
 * return SML_OK, SML_ERR_DEVICE_FAULT or SML_ERR_TIMEOUT (the SML_FAULT_*
 * bits go to *bits when bits is a host pointer); clear != 0 resets the word.
 * Allocates nothing.  (The pages have no counterpart.) */
int sml_noalloc_read_status(int clear, int32_t* bits, void* stream);

/* ---- producers: quantise new tokens and write the caches the step reads ----
 *
 * vLLM blog "vLLM 首日支持 Mistral Large 4", paragraph "可断开的 CUDA 图和融合":
 * the first round of hand-written fusions covers the indexer Q path and the
 * indexer K path, and the decode round writes the indexer K straight into the
 * FP8 cache; section "实现细节 / 模型架构": the step reads an fp8_ds_mla latent
 * cache and an FP8 indexer cache.  Reading (the pages print no quantiser):
 * a block x is stored as E4M3 codes of q = x / s, s = amax|x| / 448 (s = 1
 * when amax = 0), s and q in fp32 (IEEE division), each code the nearest E4M3
 * value to q with ties to the even code and magnitudes past 448 clamped to
 * 448.  Blocks: 128 latent values (four per row), one 128-value indexer key,
 * one query token's 64 x 128 indexer values.  Inputs must be finite.
 *
 * slot[i] = physical page * 64 + row of new token i (int32, device); -1 skips
 * the token.  A slot outside [-1, num_pages * 64) is skipped and, when
 * `workspace` is not NULL (any initialised workspace, >= 256 B), sets
 * SML_FAULT_PAGE in its status word.  Two tokens with the same slot race.
 * n = 0 is a no-op.  Rows that no slot names are left untouched. */

/* Indexer K path: k [n, 128] bf16 (16-B aligned) -> 128 e4m3 codes at
 * page*8448 + row*128 and the fp32 scale at page*8448 + 8192 + row*4. */
int sml_indexer_k_cache_write(const void* k, const int32_t* slot, int32_t n, sml_cache index_cache,
                              void* workspace, void* stream);

/* Latent write: c [n, 512] bf16 and k_pe [n, 64] bf16 (both 16-B aligned;
 * k_pe NULL for a NoPE layer, whose rows get a zero RoPE key).  By the pool's
 * format: SML_LATENT_FP8_DS_MLA -> the 656-B row at page*41984 + row*656:
 * [512 e4m3][4 fp32 block scales][64 bf16 k_pe]; SML_LATENT_E4M3 -> the 576-B
 * row at page*36864 + row*576: the codes of every value / latent.scale;
 * SML_LATENT_BF16 -> the 1,152-B row at page*73728 + row*1152: the values as
 * given (c, then k_pe). */
int sml_latent_cache_write(const void* c, const void* k_pe, const int32_t* slot, int32_t n,
                           sml_cache latent, void* workspace, void* stream);

/* Indexer Q path: iq [T, 64, 128] bf16 (16-B aligned) -> iq8 [T, 64, 128]
 * e4m3 codes (16-B aligned) and iq_scale [T] fp32, one block per token: the
 * inputs of sml_indexer_scores.  The indexer's SSMax factor is not folded in
 * here; sml_indexer_scores applies it. */
int sml_indexer_q_quant(const void* iq, int32_t num_tokens, void* iq8, float* iq_scale, void* stream);

/* ---- decode context parallelism (DCP): the cache sharded by token --------
 *
 * vLLM blog "vLLM 首日支持 Mistral Large 4", section "长上下文：解码和预填充的上下文
 * 并行", paragraph "DCP" and the list after it: the cache is sharded by token
 * over R ranks; every rank runs the indexer and top-k over its own tokens; the
 * candidates are exchanged as packed (score, id) pairs and merged with a
 * stable top-k; each rank attends over the selected tokens it holds; the
 * partial outputs are combined by their log-sum-exp.  Reading: token s of a
 * request lives on rank (s / I) % R at local position (s / (I R)) I + s % I
 * for an interleave I (I = 64 keeps a page on one rank, so a rank's shard is a
 * local block table over the same pool).  A rank's problem is the batch with
 * its local context lengths, sml_problem.vis_len = each query's local visible
 * count (its tokens among the query's n_t) and sml_problem.ssmax_len = the
 * global n_t, so that scores compare across ranks with SSMax on and any
 * number of query tokens per request.  The calls below are the steps between
 * the ranks' own sml_indexer_scores / sml_topk and their own
 * sml_sparse_mla_decode; the caller moves the arrays between GPUs (the Python
 * package's dcp module does it with torch.distributed). */
#define SML_DCP_MAX_RANKS 8

/* The ranks' top-k results (host struct; the pointers are device pointers). */
typedef struct sml_dcp_ranks {
  int32_t num_ranks;                             /* R, 1..SML_DCP_MAX_RANKS */
  int32_t interleave;                            /* I >= 1 */
  const float* scores[SML_DCP_MAX_RANKS];        /* rank r's score matrix [T, score_stride[r]] */
  int64_t score_stride[SML_DCP_MAX_RANKS];       /* its row stride (that rank's max_ctx) */
  const int32_t* idx[SML_DCP_MAX_RANKS];         /* rank r's top-k [T, topk], local positions, ascending */
  const int32_t* idx_len[SML_DCP_MAX_RANKS];     /* [T] */
  int32_t packed;  /* 1: scores[r] is [T, topk], entry i the score of candidate i (from
                      sml_dcp_pack_candidates; score_stride ignored); 0: score matrices */
} sml_dcp_ranks;

/* Pack one rank's candidates for the exchange: cand_scores [T, topk] with
 * entry i = scores[t, idx[t, i]] for i < idx_len[t], NaN past it (a NaN ranks
 * below every score).  A position outside [0, score_stride) or a length
 * outside [0, topk] gives NaN and sets SML_FAULT_INDEX / SML_FAULT_TOPK_LEN in
 * workspace (NULL or >= 256 B). */
int sml_dcp_pack_candidates(int32_t num_tokens, int32_t topk, const float* scores, int64_t score_stride,
                            const int32_t* idx, const int32_t* idx_len, float* cand_scores, void* workspace,
                            void* stream);

/* Merge: for query t, every rank's candidates (score, global position) in
 * ascending global position: merged_scores / merged_pos [T, R * topk] (row
 * stride R * topk), merged_len [T].  sml_topk over them (a problem of T
 * requests of one token, ctx_len = merged_len, max_ctx = R * topk) selects the
 * global top-k, ties to the lower global position.  workspace (NULL or >= 256
 * B) gets SML_FAULT_TOPK_LEN / SML_FAULT_INDEX for bad lengths / positions; a
 * slot that no valid candidate fills holds (NaN, -1), which ranks below every
 * score and which sml_dcp_split_selection skips (and reports).  Global
 * positions are int32: every score_stride[r] * num_ranks must fit, else
 * SML_ERR_UNSUPPORTED. */
int sml_dcp_merge_candidates(const sml_dcp_ranks* ranks, int32_t num_tokens, int32_t topk, float* merged_scores,
                             int32_t* merged_pos, int32_t* merged_len, void* workspace, void* stream);

/* Split: the selection sel [T, topk] (indices into the merged rows,
 * ascending) / sel_len [T] back to every rank's compacted list of the
 * selected tokens it holds: local_idx[r] [T, topk] (local positions,
 * ascending, -1 padded), local_len[r] [T].  local_idx / local_len are host
 * arrays of num_ranks device pointers. */
int sml_dcp_split_selection(int32_t num_ranks, int32_t interleave, int32_t num_tokens, int32_t topk,
                            const int32_t* sel, const int32_t* sel_len, const int32_t* merged_pos,
                            int32_t* const* local_idx, int32_t* const* local_len, void* workspace, void* stream);

/* LSE combine of num_parts partial attentions, each normalised by its own
 * sum: part_out[r] [T, H, 512] (16-B aligned), part_lse[r] [T, H] (host arrays
 * of device pointers) -> out [T, H, 512], lse [T, H].  A part with lse = -inf
 * drops out. */
int sml_lse_combine(int32_t num_parts, int32_t num_tokens, int32_t num_heads, const float* const* part_out,
                    const float* const* part_lse, float* out, float* lse, void* stream);

/* Synchronise `stream`, then return SML_OK, SML_ERR_DEVICE_FAULT or
 * SML_ERR_TIMEOUT from the workspace's sticky status word (its SML_FAULT_*
 * bits go to *bits when bits is a host pointer, else ignored).  clear != 0
 * resets the word. */
int sml_read_device_status(void* workspace, int clear, int32_t* bits, void* stream);

/* Static text of a status code. */
const char* sml_status_string(int code);

/* Message of the last failed call on this host thread ("" if none). */
const char* sml_last_error(void);

/* Library version, e.g. "sml 0.1.0 sm_100a". */
const char* sml_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SML_H_ */
