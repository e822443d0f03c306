/*
 * mla.h -- C ABI of the B200 (sm_100a) library for DeepSeek-V2 Multi-head Latent Attention
 * decode in absorbed form over a paged latent KV cache.
 *
 * Sources for the operations (page title, then section or figure):
 *   [A] "DeepSeek MLA, Built From the Paper", 3 Matrix absorption:
 *       q^T (W_UK c_kv) = (W_UK^T q)^T c_kv -- W_UK folds into the query; no key is rebuilt.
 *   [B] "MLA from scratch in PyTorch", The MLAAttention module / KV cache management during
 *       decode / Absorbing projections / What's not in this implementation (paged cache).
 *   [C] "Build a DeepSeek Model from Scratch", ch. 3 figures: the score is the sum of a
 *       content score and a position score; the output rearrangement applies W_UV after the
 *       weighted sum; the new latent is appended to the cache.
 *   [D] "Multi-head latent attention", Compress keys and values into one latent: each token
 *       caches c_t (width r) and one RoPE key k_rope_t (width d_r) shared by all heads.
 *
 * Conventions shared by every call:
 *   - Every data pointer is DEVICE memory owned by the caller; the library allocates nothing
 *     and never frees. Between calls it keeps only which devices already have the attention
 *     kernel's shared-memory limit raised (and, for mla_decode_static_workspace, each device's
 *     address of its workspace array). mla_decode always cuts the work into 74 ranges, one
 *     per pair of SMs of a 148-SM B200; a device with fewer SMs runs them in more than one wave.
 *   - Every call only enqueues work on `stream` (a cudaStream_t passed as void*; NULL is the
 *     legacy default stream) and returns; nothing is synchronised.
 *   - Tensors are row-major and contiguous. "dtype" tensors are float32 or bfloat16 as
 *     mla_config.dtype says; out_latent and lse are always float32; gamma is float32.
 *   - Argument and shape errors return synchronously with no launch. Data-dependent errors
 *     found on the device (a block id outside the pool, a position outside the block table,
 *     an impossible sequence length, a bounded wait that gave up) set bits in *dev_err
 *     (atomicOr) and skip the affected work; kernels never trap. The caller clears *dev_err.
 *   - Empty work (n_tokens == 0, batch == 0) returns MLA_OK without launching.
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_ABI_VERSION 8

#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, bad config value          */
  MLA_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. tensor-core decode shape)   */
  MLA_ERR_CUDA = 3,        /* a launch or runtime call failed                             */
  MLA_ERR_WORKSPACE = 4    /* workspace pointer misaligned or smaller than required       */
} mla_status;

typedef enum { MLA_F32 = 0, MLA_BF16 = 1 } mla_dtype;

/* Which kernels the calls use. AUTO: tcgen05 tensor-core kernels where dtype and shape allow
 * them -- mla_decode's attention for bf16 at H=128, r=512, d_r=64, block_size=64; the
 * projections of mla_absorb_query (d_h a multiple of 64 up to 256, r a multiple of 64) and
 * mla_output (r a multiple of 64) for bf16 -- and CUDA-core kernels otherwise. SIMT: CUDA-core
 * kernels for every call. TENSOR: tensor-core kernels, MLA_ERR_UNSUPPORTED where the shape
 * has none. (The name is historical: the choice covers every call, not only mla_decode.) */
typedef enum { MLA_DECODE_AUTO = 0, MLA_DECODE_SIMT = 1, MLA_DECODE_TENSOR = 2 } mla_decode_kernel;

typedef struct {
  int32_t num_heads;     /* H                                                    */
  int32_t head_dim;      /* d_h: width of q_nope and of each head's content key  */
  int32_t head_dim_v;    /* d_v: width of each head's value / output             */
  int32_t kv_rank;       /* r: width of the cached latent c_kv (multiple of 32)  */
  int32_t rope_dim;      /* d_r: width of the decoupled RoPE key (even, may be 0) */
  int32_t block_size;    /* tokens per cache block                               */
  float rope_base;       /* RoPE base (10000)                                    */
  float rms_eps;         /* RMSNorm epsilon (1e-6)                               */
  float softmax_scale;   /* multiplies Q . row before the softmax (1/sqrt(d_h+d_r)) */
  int32_t dtype;         /* mla_dtype of activations, weights and the cache      */
  int32_t decode_kernel; /* mla_decode_kernel                                    */
} mla_config;

/* Bits of the device error word. */
#define MLA_DEV_OOB_BLOCK 1u    /* block_table entry outside [0, num_blocks)                  */
#define MLA_DEV_OOB_POS 2u      /* sequence index or position outside the block table         */
#define MLA_DEV_WAIT_TIMEOUT 4u /* a bounded wait inside a kernel gave up; results invalid    */
#define MLA_DEV_BAD_LENGTH 8u   /* seq_lens[b] < q_per_seq or > max_blocks * block_size      */

/* Rows of the packed absorbed query and of the cache: r + d_r values. */

/*
 * mla_absorb_query -- [A], [C], [D].
 *   Q[n, h, 0:r]      = W_UK[h]^T q_nope[n, h]          (fp32 accumulation)
 *   Q[n, h, r:r+d_r]  = RoPE(q_rope[n, h], pos[n])      (adjacent pairs (2i, 2i+1) rotated by
 *                                                        pos * rope_base^(-2i/d_r))
 * q_nope (n_tokens, H, d_h) dtype; q_rope (n_tokens, H, d_r) dtype, un-rotated;
 * pos (n_tokens) int32 >= 0; w_uk (H, d_h, r) dtype -- the nn.Linear(r, H*d_h) weight,
 * rows h*d_h .. (h+1)*d_h-1 for head h, i.e. the same memory without a transpose;
 * q_out (n_tokens, H, r + d_r) dtype, rounded to nearest even when bf16.
 * The tensor-core kernel (bf16, d_h a multiple of 64 up to 256, r a multiple of 64, d_r a
 * multiple of 8, every pointer 16-byte aligned) is used where it applies. dev_err may be NULL;
 * that kernel sets MLA_DEV_WAIT_TIMEOUT in it when one of its bounded waits gives up (that
 * tile of q_out is then not written).
 */
MLA_API mla_status mla_absorb_query(const mla_config* cfg, const void* q_nope, const void* q_rope,
                            const int32_t* pos, const void* w_uk, void* q_out, int32_t n_tokens,
                            uint32_t* dev_err, void* stream);

/*
 * mla_append_latent -- [B] (norm_kv before caching; paged cache), [C] (append), [D] (row
 * layout [c_kv || k_rope]).
 *   row = [ RMSNorm(ckv_raw[n]) * gamma || RoPE(krope_raw[n], pos[n]) ]  (fp32 math, stored in
 *   dtype, bf16 rounded to nearest even), written to
 *   pool[block_table[seq_idx[n] * max_blocks + pos[n] / block_size]][pos[n] % block_size][:].
 * ckv_raw (n_tokens, r) dtype; krope_raw (n_tokens, d_r) dtype; gamma (r) float32;
 * seq_idx, pos (n_tokens) int32; block_table (batch, max_blocks) int32;
 * pool (num_blocks, block_size, r + d_r) dtype. A row whose sequence index or position is
 * outside the table sets MLA_DEV_OOB_POS, one whose block id is outside the pool sets
 * MLA_DEV_OOB_BLOCK; neither is written. No other pool byte is touched.
 */
MLA_API mla_status mla_append_latent(const mla_config* cfg, const void* ckv_raw, const void* krope_raw,
                             const float* gamma, const int32_t* seq_idx, const int32_t* pos,
                             const int32_t* block_table, int32_t batch, int32_t max_blocks,
                             void* pool, int32_t num_blocks, int32_t n_tokens, uint32_t* dev_err,
                             void* stream);

/*
 * Workspace of mla_decode in bytes for this configuration and batch shape (0 when the
 * configuration is invalid). The workspace holds the split-KV schedule and the partial
 * outputs of sequences split across work ranges; it must be 256-byte aligned.
 */
MLA_API size_t mla_decode_workspace_size(const mla_config* cfg, int32_t batch, int32_t q_per_seq);

/*
 * mla_decode -- split-KV flash decoding in absorbed form ([A], [B] Absorbing projections:
 * attend directly to latents; [C] score = content + position).
 * For sequence b, query token t (bt = b * q_per_seq + t) and head h, with
 * L = seq_lens[b] - q_per_seq + 1 + t rows attended (rows 0 .. L-1: causal among the new
 * tokens, each new token sees itself):
 *   s_j = softmax_scale * Q[bt, h, :] . row_j,   p = softmax(s),
 *   out_latent[bt, h, :] = sum_j p_j row_j[0:r],  lse[bt, h] = log(sum_j exp(s_j)).
 * q (batch * q_per_seq, H, r + d_r) dtype; pool and block_table as in mla_append_latent;
 * seq_lens (batch) int32: rows valid after this step's append (callers advance it by
 * q_per_seq before the call); out_latent (batch * q_per_seq, H, r) float32;
 * lse (batch * q_per_seq, H) float32 or NULL. q, pool and out_latent must be 16-byte aligned
 * (MLA_ERR_INVALID_ARG otherwise). Runs three stages on `stream`: a one-CTA
 * planner that cuts all (sequence, token) row ranges into equal 64-row chunks of work, the
 * attention kernel, and a log-sum-exp combine of sequences that were split. A length outside
 * [1, max_blocks * block_size] sets MLA_DEV_BAD_LENGTH and that row's output is 0 (lse -inf).
 * Deterministic: the same inputs give the same bits.
 */
MLA_API mla_status mla_decode(const mla_config* cfg, const void* q, const void* pool,
                      const int32_t* block_table, int32_t max_blocks, int32_t num_blocks,
                      const int32_t* seq_lens, int32_t batch, int32_t q_per_seq, void* workspace,
                      size_t workspace_bytes, float* out_latent, float* lse, uint32_t* dev_err,
                      void* stream);

/* Stages of mla_decode, for timing them apart: a bit mask of the stages to enqueue.
 * Running PLAN, then ATTEND, then COMBINE (in order, same arguments) equals mla_decode. */
#define MLA_STAGE_PLAN 1
#define MLA_STAGE_ATTEND 2
#define MLA_STAGE_COMBINE 4
MLA_API mla_status mla_decode_stages(const mla_config* cfg, int32_t stages, const void* q,
                             const void* pool, const int32_t* block_table, int32_t max_blocks,
                             int32_t num_blocks, const int32_t* seq_lens, int32_t batch,
                             int32_t q_per_seq, void* workspace, size_t workspace_bytes,
                             float* out_latent, float* lse, uint32_t* dev_err, void* stream);

/*
 * Size of the device array that mla_decode_static_workspace uses as its workspace: 40 MiB,
 * enough for the DeepSeek-V2 shape (H = 128, r = 512) at any batch up to several thousand
 * (query token, sequence) pairs.
 */
#define MLA_STATIC_WORKSPACE_BYTES (40u << 20)

/*
 * mla_decode_static_workspace -- no counterpart on the pages: a library-side addition.
 * Exactly mla_decode (same arguments, same kernels, same results) without the workspace
 * arguments, for callers that cannot allocate device memory themselves: a host program with
 * no device allocator of its own, or a decode loop that must not call cudaMalloc because it
 * synchronises the device. The workspace is a file-scope device array of
 * MLA_STATIC_WORKSPACE_BYTES that every GPU loading the library holds until exit. This call
 * allocates nothing (no cudaMalloc, no cudaFree, no allocating library routine).
 *   - Returns MLA_ERR_WORKSPACE when mla_decode_workspace_size(cfg, batch, q_per_seq) exceeds
 *     MLA_STATIC_WORKSPACE_BYTES; nothing is launched.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 *     with that device current; make that first call before any stream capture.
 *   - All calls share the one array, which keeps the last call's contents: calls that overlap
 *     on the GPU (other streams, other threads) race and must be serialised by the caller.
 */
MLA_API mla_status mla_decode_static_workspace(const mla_config* cfg, const void* q,
                                               const void* pool, const int32_t* block_table,
                                               int32_t max_blocks, int32_t num_blocks,
                                               const int32_t* seq_lens, int32_t batch,
                                               int32_t q_per_seq, float* out_latent, float* lse,
                                               uint32_t* dev_err, void* stream);

/*
 * mla_output -- [B] Absorbing projections, [C] the output rearrangement figure (W_UV applied
 * after the weighted sum): o[n, h, :] = W_UV[h] out_latent[n, h, :] (fp32 accumulation).
 * out_latent (n_tokens, H, r) float32; w_uv (H, d_v, r) dtype (the nn.Linear(r, H*d_v)
 * weight); o (n_tokens, H, d_v) dtype. W_O is not part of the library.
 * For bf16 the tensor-core kernel feeds out_latent to its bf16 MMA as two terms, hi = bf16(x)
 * and lo = bf16(x - hi) (about 16 significant bits of x); the products are summed in fp32.
 * The tensor-core kernel is used only when out_latent and w_uv are 16-byte aligned.
 * dev_err may be NULL; it receives MLA_DEV_WAIT_TIMEOUT as for mla_absorb_query.
 */
MLA_API mla_status mla_output(const mla_config* cfg, const float* out_latent, const void* w_uv, void* o,
                      int32_t n_tokens, uint32_t* dev_err, void* stream);

/*
 * mla_decode_step -- one whole decode step: exactly mla_absorb_query, mla_append_latent,
 * mla_decode and mla_output called in that order with these arguments (the sources of each are
 * cited above), for n = batch * q_per_seq new tokens, token k = b * q_per_seq + t being query
 * token t of sequence b:
 *   mla_absorb_query(cfg, q_nope, q_rope, pos, w_uk, q_work, n)
 *   mla_append_latent(cfg, ckv_raw, krope_raw, gamma, seq_idx, pos, block_table, batch,
 *                     max_blocks, pool, num_blocks, n)
 *   mla_decode(cfg, q_work, pool, block_table, max_blocks, num_blocks, seq_lens, batch,
 *              q_per_seq, workspace, workspace_bytes, out_latent, lse)
 *   mla_output(cfg, out_latent, w_uv, o, n)
 * so pos and seq_idx are the new tokens' positions and sequences, and seq_lens already counts
 * the new rows. q_work (n, H, r + d_r) dtype receives the absorbed query. The results (q_work,
 * the pool's new rows, out_latent, lse, o, *dev_err) are bit for bit those of the four calls.
 * Every argument is validated as the four calls validate theirs before anything is enqueued
 * (the same status codes). Where the tensor-core kernels apply to every stage (bf16, the
 * attention kernel's shape, 16-byte aligned operands) the step takes four launches instead of
 * six: the absorbed query, the append and the decode planner run as parts of one grid (they do
 * not depend on one another), followed by the attention, the combine and the output
 * projection; otherwise the four calls' own kernels run in order.
 */
MLA_API mla_status mla_decode_step(const mla_config* cfg, const void* q_nope, const void* q_rope,
                                   const void* w_uk, const void* ckv_raw, const void* krope_raw,
                                   const float* gamma, const int32_t* seq_idx, const int32_t* pos,
                                   const int32_t* block_table, int32_t max_blocks, void* pool,
                                   int32_t num_blocks, const int32_t* seq_lens, int32_t batch,
                                   int32_t q_per_seq, void* q_work, void* workspace,
                                   size_t workspace_bytes, float* out_latent, float* lse,
                                   const void* w_uv, void* o, uint32_t* dev_err, void* stream);

/*
 * The decode front end: hidden states x -> the four per-token inputs of the calls above
 * ([B] The MLAAttention module: c_q = RMSNorm(W_DQ x), q = W_UQ c_q; [D] the RoPE query and
 * the shared RoPE key are projected from x; c_kv = W_DKV x, normalised at append).
 */
typedef struct {
  int32_t d_model;  /* hidden size: the K of every product with x                          */
  int32_t q_rank;   /* query latent width r_q; 0 for a full-rank query (q_nope = W_Q x)     */
  float q_rms_eps;  /* eps of the RMSNorm of c_q                                            */
} mla_front_config;

/* Workspace of mla_project in bytes (0 for an invalid configuration); 256-byte aligned. */
MLA_API size_t mla_project_workspace_size(const mla_config* cfg, const mla_front_config* front,
                                          int32_t n_tokens);

/*
 * mla_project -- for n_tokens tokens x (n_tokens, d_model) dtype, with weights in the
 * nn.Linear layout (out_features, d_model or q_rank) dtype:
 *   q_rank > 0:  c_q = W_DQ x (w_dq: (q_rank, d_model)), c_q' = c_q / sqrt(mean(c_q^2) + eps)
 *                * gamma_q (fp32 statistics; gamma_q (q_rank) float32), stored in dtype;
 *                q_nope = W_UQ c_q' (w_uq: (H * d_h, q_rank));
 *   q_rank == 0: q_nope = W_Q x (w_dq holds W_Q: (H * d_h, d_model)); gamma_q, w_uq unused;
 *   q_rope = W_QR x (w_qr: (H * d_r, d_model)), ckv_raw = W_DKV x (w_dkv: (r, d_model)),
 *   krope_raw = W_KR x (w_kr: (d_r, d_model)); with d_r == 0, w_qr, w_kr, q_rope and
 *   krope_raw are unused.
 * Outputs q_nope (n, H, d_h), q_rope (n, H, d_r), ckv_raw (n, r), krope_raw (n, d_r), dtype:
 * the inputs of mla_absorb_query and mla_append_latent. Products accumulate in fp32 and are
 * rounded once. bf16 with d_model and q_rank multiples of 8 runs on the tensor cores (x and
 * every weight 16-byte aligned); fp32 on CUDA cores; bf16 with other widths returns
 * MLA_ERR_UNSUPPORTED. Deterministic. q_rank at most
 * 12288, d_model at most 57344. dev_err may be NULL (MLA_DEV_WAIT_TIMEOUT as elsewhere).
 */
MLA_API mla_status mla_project(const mla_config* cfg, const mla_front_config* front,
                               const void* x, const void* w_dq, const float* gamma_q,
                               const void* w_uq, const void* w_qr, const void* w_dkv,
                               const void* w_kr, void* q_nope, void* q_rope, void* ckv_raw,
                               void* krope_raw, int32_t n_tokens, void* workspace,
                               size_t workspace_bytes, uint32_t* dev_err, void* stream);

/* Workspace of mla_prefill in bytes (0 for an invalid configuration); 256-byte aligned. */
MLA_API size_t mla_prefill_workspace_size(const mla_config* cfg, int32_t n_tokens);

/*
 * mla_prefill -- causal self-attention of prompts in the expanded form ([B] The MLAAttention
 * module: K and V rebuilt from every cached latent, the causal mask when S > 1; the expanded
 * form takes d_h + d_r multiply-adds per score against r + d_r absorbed, so it is the cheaper
 * one when every key serves many queries). For a batch of prompts packed one after another
 * (sequence b holds tokens cu_seqlens[b] .. cu_seqlens[b + 1] - 1) and every head h:
 *   K[j, h] = [W_UK[h] c_kv[j] ‖ k_rope[j]],  V[j, h] = W_UV[h] c_kv[j],
 *   Q[i, h] = [q_nope[i, h] ‖ RoPE(q_rope[i, h], pos[i])],
 *   o[i, h] = sum_j p_j V[j, h],  p = softmax_j(softmax_scale * Q[i, h] . K[j, h])
 * over the keys j of i's sequence with j <= i.
 * q_nope (n, H, d_h), q_rope (n, H, d_r) before rotation, pos (n) int32, rows (n, r + d_r):
 * the tokens' cache rows [RMSNorm(c_kv) * gamma ‖ RoPE(k_rope)] as mla_append_latent writes
 * them, here contiguous; w_uk (H, d_h, r), w_uv (H, d_v, r); cu_seqlens (batch + 1) int32 on
 * the device, non-decreasing from 0 to n; max_seqlen >= every sequence's length (host value);
 * o (n, H, d_v). All dtype. bf16 with d_h = d_v = 128, d_r = 64 runs on the tensor cores
 * (every pointer 16-byte aligned); other shapes and fp32 on CUDA cores (d_v <= 256).
 */
MLA_API mla_status mla_prefill(const mla_config* cfg, const void* q_nope, const void* q_rope,
                               const int32_t* pos, const void* rows, const void* w_uk,
                               const void* w_uv, const int32_t* cu_seqlens, int32_t batch,
                               int32_t max_seqlen, int32_t n_tokens, void* o, void* workspace,
                               size_t workspace_bytes, uint32_t* dev_err, void* stream);

/*
 * FP8 latent cache ("MLA from scratch in PyTorch", What's not in this implementation: the
 * latent cache can be quantised to FP8). A pool row is r + d_r e4m3 codes (one byte each,
 * (num_blocks, block_size, r + d_r) uint8) with one float32 scale per row
 * (row_scale: (num_blocks, block_size)); the row reads back as code_j * scale.
 *
 * mla_append_latent_fp8 -- mla_append_latent's row y = [RMSNorm(c_kv) * gamma ‖ RoPE(k_rope)]
 * (fp32), stored as scale = max_j |y_j| / 448 (1 for an all-zero row) and
 * code_j = e4m3(y_j / scale), rounded to nearest even and saturated at 448. Arguments as
 * mla_append_latent, with the fp8 pool and its row_scale.
 */
MLA_API mla_status mla_append_latent_fp8(const mla_config* cfg, const void* ckv_raw,
                                         const void* krope_raw, const float* gamma,
                                         const int32_t* seq_idx, const int32_t* pos,
                                         const int32_t* block_table, int32_t batch,
                                         int32_t max_blocks, uint8_t* pool, float* row_scale,
                                         int32_t num_blocks, int32_t n_tokens, uint32_t* dev_err,
                                         void* stream);

/* Workspace of mla_decode_fp8 in bytes (0 for an invalid configuration); 256-byte aligned. */
MLA_API size_t mla_decode_fp8_workspace_size(const mla_config* cfg, int32_t batch,
                                             int32_t q_per_seq, int32_t max_blocks);

/*
 * mla_decode_fp8 -- mla_decode over an fp8 pool: every row j of the attention is
 * code_j * row_scale[j]. Arguments and results as mla_decode (q in the config's dtype), with
 * the fp8 pool, its row_scale and a workspace of mla_decode_fp8_workspace_size bytes. Where
 * mla_decode would take the tensor-core attention (bf16, its shape), the step's blocks are
 * first expanded to bf16 in the workspace (batch x max_blocks blocks of scratch, rounded to
 * nearest even) and that kernel runs over them; otherwise the CUDA-core attention reads the
 * codes directly (fp32 arithmetic).
 */
MLA_API mla_status mla_decode_fp8(const mla_config* cfg, const void* q, const uint8_t* pool,
                                  const float* row_scale, const int32_t* block_table,
                                  int32_t max_blocks, int32_t num_blocks, const int32_t* seq_lens,
                                  int32_t batch, int32_t q_per_seq, void* workspace,
                                  size_t workspace_bytes, float* out_latent, float* lse,
                                  uint32_t* dev_err, void* stream);

/* Most parts mla_combine_partials merges in one call. */
#define MLA_MAX_COMBINE_PARTS 256

/*
 * mla_combine_partials -- merge partial decode results of the same row groups computed over
 * disjoint sets of each sequence's cache rows: the per-GPU results of a context-parallel
 * split, where every GPU holds a contiguous slice of each sequence's rows, runs mla_decode on
 * its slice, and the slices' (out_latent, lse) are gathered. The merge is the one mla_decode
 * applies to its own work ranges: a softmax over all rows equals the softmaxes over disjoint
 * row sets weighted by their shares of the normaliser ([B] Absorbing projections: attend
 * directly to latents; "MLA from scratch in PyTorch", Memory comparison: the cache of long
 * contexts outgrows one GPU). For row group k < n and head h:
 *   L = log(sum_i exp(part_lse[i, k, h])),
 *   out_latent[k, h, :] = sum_i exp(part_lse[i, k, h] - L) * part_latent[i, k, h, :],
 *   lse[k, h] = L.
 * part_latent (parts, n, H, r) float32 and part_lse (parts, n, H) float32, part-major, each
 * part as mla_decode writes out_latent and lse; out_latent (n, H, r) float32; lse (n, H)
 * float32 or NULL. part_latent and out_latent must be 16-byte aligned; out_latent must not
 * overlap the parts. 1 <= parts <= MLA_MAX_COMBINE_PARTS. A part whose lse is -inf holds no
 * rows and is skipped (its part_latent is not read); a row group with no rows in any part gets
 * 0 and lse -inf. fp32 arithmetic in part order: the same inputs give the same bits.
 * MLA_ERR_INVALID_ARG for a bad config, a null pointer, misalignment or parts out of range;
 * n == 0 returns MLA_OK without launching.
 */
MLA_API mla_status mla_combine_partials(const mla_config* cfg, const float* part_latent,
                                        const float* part_lse, int32_t parts, int32_t n,
                                        float* out_latent, float* lse, void* stream);

/* Human-readable name of a status code (static storage). */
MLA_API const char* mla_status_string(mla_status status);

/* MLA_ABI_VERSION of the built library. */
MLA_API int32_t mla_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MLA_H_ */
