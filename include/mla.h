/*
 * mla.h — C ABI of libmla: Multi-head Latent Attention (MLA) decode over a latent KV cache
 * on NVIDIA B200 (sm_100a).
 *
 * The method (pages cited by title and section):
 *   "DeepSeek-V2 大模型论文原文 PDF" (hncyxsy.com), section 2.1: every token is compressed to a
 *   latent c_KV = W_DKV h (d_c values); K and V are its up-projections W_UK c_KV, W_UV c_KV.
 *   Section 2.2: W_UK is absorbed into the query and W_UV into the output, so K and V are
 *   never formed.  Section 2.3: a decoupled RoPE key (d_rope values, shared by all heads)
 *   is cached beside the latent.  "从一份技术报告说起：DeepSeek 2025 到底在做什么"
 *   (m.nlpx.cn), section 3.3: 512 + 64 = 576 cached values per token.
 *
 * Conventions shared by every call
 *   - Every pointer argument is a DEVICE pointer owned by the caller, except `dims` and
 *     `cache` (host structs read during the call).  The library never allocates or frees
 *     memory; scratch space ("workspace") is passed in by the caller and its size is
 *     returned by the matching *_workspace_size query.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls enqueue work on it
 *     and return without synchronising.  The current CUDA device must own all pointers.
 *   - Argument errors are detected on the host, return MLA_ERR_INVALID_ARG or
 *     MLA_ERR_UNSUPPORTED and enqueue nothing.  A launch failure returns MLA_ERR_CUDA.
 *   - Data errors only visible on the device (a page id outside [0, num_pages), a
 *     position outside the RoPE table) are not faults: the kernel skips the access and
 *     records the first such error in a per-device error word, read and cleared by
 *     mla_check_device_error().
 *   - The library caches, per device, the device addresses of its own static buffers (the
 *     error word, the no-allocation scratch).  Do not keep using it across a
 *     cudaDeviceReset (or anything else that destroys the device's primary context) in the
 *     same process: those cached addresses would be stale.
 *   - Tensors are dense, row-major, innermost dimension last, with the shapes given.
 *   - "act" dtype (dims.act_dtype) is the dtype of h, q, weights, o_lat and outputs:
 *     MLA_F32 or MLA_BF16.  Accumulation is always fp32.
 *   - Overlap of consecutive calls (bf16 tensor-core path): the projection kernels of
 *     mla_append_cache, mla_absorb_query and mla_output_up are launched with programmatic
 *     stream serialization, and the preceding library kernel on the stream lets them start
 *     early.  Before waiting for that kernel to complete they read only their weights
 *     (w_dkv, w_kr, w_uk, w_uv), and q_nope in mla_absorb_query; everything else
 *     they read, and everything they write, comes after the wait.  So a weight (or query
 *     input) must not be an output of the immediately preceding library call on the same
 *     stream.  Setting MLA_PDL=0 in the environment (read once) launches them normally.
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1, /* null pointer, bad size, inconsistent dims */
  MLA_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. d_c not a multiple of 128 for FP8) */
  MLA_ERR_CUDA = 3,        /* a CUDA runtime call failed (launch error, no device) */
  MLA_ERR_DEVICE = 4,      /* mla_check_device_error: a kernel recorded a data error */
  MLA_ERR_TIMEOUT = 5      /* mla_check_device_error: a bounded device wait gave up */
} mla_status;

typedef enum { MLA_F32 = 0, MLA_BF16 = 1, MLA_FP8_E4M3 = 2 } mla_dtype;

/* Model dimensions.  page_size is the number of tokens per cache page (64 for the
 * tensor-core decode; any value >= 1 for the general one).  scale multiplies the scores
 * (1/sqrt(d_nope + d_rope) is the usual choice).  d_v is the per-head output width of W_UV. */
typedef struct {
  int32_t d_model, d_c, d_rope, d_nope, d_v, n_heads, page_size;
  int32_t act_dtype;   /* mla_dtype: MLA_F32 or MLA_BF16 */
  int32_t cache_dtype; /* mla_dtype: MLA_F32 (act F32 only), MLA_BF16, MLA_FP8_E4M3 */
  float scale;
} mla_dims;

/* A paged latent cache ("DeepSeek大模型核心技术解析" (intelliparadigm.com), section 6.1: blocked
 * KV storage).  Token p of sequence b lives in page block_table[b * max_pages_per_seq +
 * p / page_size], slot p % page_size.
 *   cache_dtype F32/BF16: rows   = [num_pages, page_size, d_c + d_rope], one row is
 *                                  c_KV (d_c values) followed by the rotated k_rope.
 *   cache_dtype FP8_E4M3: rows   = [num_pages, page_size, d_c] uint8 E4M3 codes of c_KV,
 *                         scales = [num_pages, page_size, d_c / 128] fp32, one scale per
 *                                  128-value block (value = code * scale),
 *                         rope   = [num_pages, page_size, d_rope] bf16 rotated k_rope.
 *   (FP8 KV cache with per-block scales: intelliparadigm.com section 6.3; "8.1 DeepSeek
 *   架构：MLA、DeepSeekMoE 与 FP8 训练" (hdu-wiki.cn) section 5.) */
typedef struct {
  void* rows;
  float* scales;
  void* rope;
  const int32_t* block_table; /* [num_seqs, max_pages_per_seq] int32 page ids */
  int32_t max_pages_per_seq;
  int32_t num_pages;          /* pages in the pool; valid ids are 0 .. num_pages-1 */
  int32_t num_seqs;           /* rows of block_table */
} mla_cache;

/* ---------------------------------------------------------------------------------------
 * mla_rope_table — precomputed RoPE cos/sin ("从一份技术报告说起" (m.nlpx.cn), section 5.2).
 * cos_out/sin_out: [max_pos, d_rope / 2] fp32; entry [p][i] = cos/sin(p * theta^(-2i/d_rope)),
 * evaluated in fp64 and rounded once.  Pairs (x[2i], x[2i+1]) of a RoPE vector are rotated by
 * angle [p][i].  Errors: d_rope odd or <= 0, max_pos <= 0, theta <= 0, null pointers. */
MLA_API mla_status mla_rope_table(int32_t d_rope, int32_t max_pos, float theta, float* cos_out,
                          float* sin_out, void* stream);

/* ---------------------------------------------------------------------------------------
 * mla_append_cache — step 1: compress new tokens into the cache
 * ("DeepSeek-V2 大模型论文原文 PDF" sections 2.1 and 2.3; hdu-wiki.cn section 2).
 * For token t: c = W_DKV h[t] (d_c), k = RoPE_{pos[t]}(W_KR h[t]) (d_rope), then stored as
 * act-precision rows (F32/BF16, round to nearest even) or as E4M3 codes with one fp32
 * scale per 128-value block (s = amax/448, s = 1 for an all-zero block) into the page of
 * (seq_idx[t], pos[t]).
 *   h:        [n_tok, d_model] act dtype
 *   seq_idx:  [n_tok] int32, sequence of each token (row of the block table)
 *   pos:      [n_tok] int32, position of each token (0-based, < rope_rows)
 *   w_dkv:    [d_c, d_model] act dtype;  w_kr: [d_rope, d_model] act dtype
 *   rope_cos, rope_sin: [rope_rows, d_rope/2] fp32 (from mla_rope_table)
 *   workspace: fp32 scratch of mla_append_workspace_size(dims, n_tok) bytes (may be NULL
 *              when that size is 0).  The size is 0 on the bf16 tensor-core path (bf16
 *              activations, d_model % 64 == 0, d_c % 128 == 0, d_rope <= 128): one kernel
 *              computes both projections, reduces its split-K partial sums on chip in a fixed
 *              order (the result does not depend on timing) and writes the cache.  That path
 *              needs h, w_dkv, w_kr and the cache arrays 16-byte aligned (MLA_ERR_UNSUPPORTED
 *              otherwise).
 * A token whose seq_idx, pos or page id is out of range is skipped and reported through
 * the device error word.  Two tokens writing the same (sequence, position) race; the caller
 * avoids that.  n_tok == 0 is a no-op. */
MLA_API size_t mla_append_workspace_size(const mla_dims* dims, int32_t n_tok);
MLA_API mla_status mla_append_cache(const mla_dims* dims, const void* h, int32_t n_tok,
                            const int32_t* seq_idx, const int32_t* pos, const void* w_dkv,
                            const void* w_kr, const float* rope_cos, const float* rope_sin,
                            int32_t rope_rows, const mla_cache* cache, void* workspace,
                            size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * mla_absorb_query — step 2: fold W_UK into the query ("DeepSeek-V2 大模型论文原文 PDF" 2.2).
 * q_packed[t, h] = ( W_UK[h]^T q_nope[t, h]  ||  RoPE_{q_pos[t]}(q_rope[t, h]) ).
 *   q_nope:  [n_tok, H, d_nope] act;  q_rope: [n_tok, H, d_rope] act;  q_pos: [n_tok] int32
 *   w_uk:    [H, d_nope, d_c] act (head h's block of the [H*d_nope, d_c] up-projection)
 *   q_packed:[n_tok, H, d_c + d_rope] act (output)
 * On the bf16 tensor-core path (d_c <= 1024, d_nope <= 256, d_rope % 32 == 0) one kernel per
 * call does the GEMM and the RoPE when q_rope, q_packed and the RoPE tables are 16-byte
 * aligned; otherwise a GEMM and a RoPE kernel.  A q_pos outside the table is reported through
 * the device error word and that token's q_rope is copied unrotated.
 * n_tok == 0 is a no-op. */
MLA_API mla_status mla_absorb_query(const mla_dims* dims, const void* q_nope, const void* q_rope,
                            const int32_t* q_pos, int32_t n_tok, const void* w_uk,
                            const float* rope_cos, const float* rope_sin, int32_t rope_rows,
                            void* q_packed, void* stream);

/* ---------------------------------------------------------------------------------------
 * mla_decode_attention — step 3 (+ step 4, the split combine): attention over the latent
 * cache in the absorbed form ("DeepSeek-V2 大模型论文原文 PDF" 2.2-2.3; the softmax attention of
 * intelliparadigm.com section 3.3).  For query row (b, j, h):
 *   s_p = (q_lat . c_p + q_rope . k_p) * scale  over the attended cached tokens p,
 *   o_lat = sum_p softmax(s)_p c_p,   lse = log sum_p exp(s_p).
 * Query token j of sequence b (j < s_q) sits at position seq_lens[b] - s_q + j.  causal = 0:
 * every query attends all seq_lens[b] cached tokens; causal = 1: it attends positions
 * <= its own.  A query with nothing to attend gets o_lat = 0, lse = -inf.
 *   q_packed: [batch * s_q, H, d_c + d_rope] act (from mla_absorb_query), row = b * s_q + j
 *   seq_lens: [batch] int32 cached tokens per sequence (0 <= L <= max_pages_per_seq * page)
 *   n_split:  KV chunks per sequence (split-KV) on the general path: each query row's pages are
 *             cut into n_split equal ranges (0 lets the library pick a count).  The tensor-core
 *             path ignores it and always cuts the pages of all sequences, concatenated, into
 *             max(1, 74 / s_q) equal ranges, each walked by s_q persistent clusters (one per SM
 *             pair and query token, the s_q tokens of a sequence side by side so that each
 *             page is read from memory once), so every SM gets the same number of pages
 *             whatever the length mix.  Rows covered by more than one range write partial
 *             (o, lse) to the workspace and a log-sum-exp combine kernel merges them.
 *   workspace: scratch of mla_decode_workspace_size(...) bytes for the same arguments (on the
 *             tensor-core path 146 partial slots of H x (d_c + 1) fp32, about 39 MB at 128
 *             heads, plus 8 bytes per query row).
 *   o_lat:    [batch * s_q, H, d_c] act (output);  lse: [batch * s_q, H] fp32 (output, may be NULL)
 * Supported: d_c + d_rope <= 576; the tensor-core path needs BF16 activations, a BF16 or FP8
 * cache, page_size 64, d_c = 512, d_rope = 64, n_heads <= 128, and 16-byte aligned q_packed,
 * o_lat and cache arrays (misaligned arrays give MLA_ERR_UNSUPPORTED); other shapes take the
 * general path.  With at most 16 heads and a BF16 cache a small-head tensor-core kernel runs
 * instead (warp-level MMAs, 16 head rows, two persistent CTAs per SM on the same partition,
 * 590 partial slots).
 * Precision on the tensor-core path: the scores are fp32 sums over all 576 dims of products of
 * the bf16 inputs (any finite bf16 range; only the fp32 range bounds the scores), the softmax
 * runs in fp32 against a running maximum (P <= 2^8 before rounding), P is rounded to bf16 (fp16
 * on an FP8 cache) for the P.V product, and O accumulates in fp32.  On an FP8 cache each latent value code * scale is
 * rounded once to fp16, and Q's latent half is rounded to fp16 (saturating at 65504), so that
 * path needs |q|, |c| below 65504; the rope part stays bf16. */
MLA_API size_t mla_decode_workspace_size(const mla_dims* dims, int32_t batch, int32_t s_q,
                                 int32_t n_split, int32_t max_pages_per_seq);
MLA_API mla_status mla_decode_attention(const mla_dims* dims, const void* q_packed,
                                const mla_cache* cache, const int32_t* seq_lens, int32_t batch,
                                int32_t s_q, int32_t causal, int32_t n_split, void* workspace,
                                size_t workspace_bytes, void* o_lat, float* lse, void* stream);

/* ---------------------------------------------------------------------------------------
 * mla_output_up — step 5: W_UV on the output side ("DeepSeek-V2 大模型论文原文 PDF" 2.2).
 * out[t, h] = W_UV[h] o_lat[t, h].
 *   o_lat: [n_tok, H, d_c] act;  w_uv: [H, d_v, d_c] act;  out: [n_tok, H, d_v] act
 * n_tok == 0 is a no-op. */
MLA_API mla_status mla_output_up(const mla_dims* dims, const void* o_lat, int32_t n_tok,
                         const void* w_uv, void* out, void* stream);

/* ---------------------------------------------------------------------------------------
 * mla_decode_attention_noalloc — mla_decode_attention for callers that cannot allocate.
 * The pages have no counterpart: this is an engineering entry point of the library.
 *
 * Some callers cannot hand the library scratch memory: code that runs inside a host
 * framework which owns every device allocation (a fixed memory budget or its own pool)
 * and gives plug-ins no allocator, or latency-critical paths where a cudaMalloc/cudaFree
 * would synchronise the device.  This variant keeps the split-KV partials in a
 * file-scope static device buffer of MLA_NOALLOC_SCRATCH_BYTES inside the library, so the
 * caller passes only inputs and outputs.  It calls no cudaMalloc, cudaFree or other
 * allocating routine.
 *   - Every GPU that loads the library holds the buffer (64 MiB) until the process exits.
 *   - Arguments and results are those of mla_decode_attention without the workspace.
 *   - A request whose partials need more than MLA_NOALLOC_SCRATCH_BYTES (see
 *     mla_decode_workspace_size for the same arguments) returns MLA_ERR_UNSUPPORTED and
 *     enqueues nothing; lower n_split or split the batch.  On the tensor-core path (at most
 *     128 heads) the partials never exceed 146 slots (39 MB at 128 heads) plus 8 bytes per
 *     query row, so only a batch of millions of rows is refused there.
 *   - The first call on a device looks up the buffer's device address (once per device,
 *     with that device current); make that first call before any stream capture.
 *   - All calls on a device share the one buffer, which keeps the last call's contents.
 *     Nothing in it needs to start at zero (each call writes every partial it reads), but
 *     calls that overlap on the GPU (different streams, or different host threads) race on
 *     it: serialise them. */
#define MLA_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
MLA_API mla_status mla_decode_attention_noalloc(const mla_dims* dims, const void* q_packed,
                                                const mla_cache* cache, const int32_t* seq_lens,
                                                int32_t batch, int32_t s_q, int32_t causal,
                                                int32_t n_split, void* o_lat, float* lse,
                                                void* stream);

/* ---------------------------------------------------------------------------------------
 * Status helpers. */
MLA_API const char* mla_status_string(mla_status s);
/* Synchronises `stream`, then reads and clears the current device's error word.
 * Returns MLA_OK, MLA_ERR_DEVICE (a bad page id or position was skipped, or a kernel found
 * its dynamic shared memory misaligned and computed nothing: kind 5), MLA_ERR_TIMEOUT (a
 * bounded wait inside a kernel gave up) or MLA_ERR_CUDA.
 * If detail is not NULL it receives the raw error word (kind << 24 | first bad value). */
MLA_API mla_status mla_check_device_error(void* stream, int32_t* detail);
/* Library version as major * 10000 + minor * 100 + patch. */
MLA_API int32_t mla_version(void);
/* Number of CUDA kernels this process has launched through the library so far (all
 * devices, all threads).  For profiling and launch accounting; never resets. */
MLA_API uint64_t mla_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* MLA_H_ */
