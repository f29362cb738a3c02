/*
 * mla.h — C ABI of the absorbed Multi-head Latent Attention decode library (libmla.so).
 *
 * One decode step of one attention layer whose cache keeps, per position, only a latent row
 * c = RMSNorm(x·W_DKV) of width d_c and one RoPE key k_r = RoPE(x·W_KR) of width d_r shared by all
 * heads (« L'attention latente : compresser le cache », sections « L'idée : garder un résumé » and
 * « L'obstacle : RoPE »). Queries are absorbed into latent space and attend the cached rows
 * directly (same page, « Ce que DeepSeek fait de plus »; « Résumé technique : GQLA … »,
 * « Chemin MQA-Absorbé »). The grouped GQA path of the GQLA page (« Chemin GQA ») is also here.
 *
 * Conventions shared by every call
 *  - Pointers named as tensors are DEVICE pointers owned by the caller. The library never
 *    allocates, frees or synchronises: it validates the arguments on the host, then enqueues
 *    kernels on `stream` (a cudaStream_t; NULL = the legacy default stream) and returns.
 *  - Row-major layouts; shapes are written [outer, ..., inner]. Every tensor pointer must be
 *    16-byte aligned and every row stride a multiple of 16 bytes.
 *  - dtype is MLA_F32 or MLA_BF16; it is the storage type of the cache, weights, queries and
 *    outputs of that call. Accumulation, softmax and normalisation are fp32 in every kernel.
 *  - B sequences with s_q new tokens each: B * s_q must not exceed INT32_MAX (else
 *    MLA_ERR_INVALID_ARG).
 *  - seqlens[b] counts the cached positions of sequence b INCLUDING this step's s_q new tokens;
 *    new token t (0 <= t < s_q) sits at position seqlens[b] - s_q + t and attends positions
 *    0 .. seqlens[b] - s_q + t (causal among the new tokens).
 *  - Paged cache: position p of sequence b lives in page block_table[b*max_pages + p/page_size],
 *    slot p % page_size; page_size is 64. Row r = page*64 + slot of a pool starts at
 *    base + r*stride elements.
 *  - Return value: MLA_OK or an error code. Argument errors (MLA_ERR_INVALID_ARG,
 *    MLA_ERR_UNSUPPORTED, MLA_ERR_WORKSPACE) are found on the host before anything is enqueued.
 *    MLA_ERR_CUDA reports a failed CUDA call (a launch, a kernel attribute); in a call that
 *    enqueues several kernels it may follow the earlier ones, and the call's outputs are then
 *    undefined. Errors found on the device (a page id outside the pool, a wait that timed out)
 *    are recorded in a per-device status word that mla_check_status() reads; the offending
 *    access is skipped, never performed.
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The library exports these calls only (it is built with hidden visibility): two builds loaded in
 * one process never share internal state. */
#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

enum mla_status {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer or stride */
  MLA_ERR_UNSUPPORTED = 2,   /* valid arguments the library has no kernel for (dtype, shape) */
  MLA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than the matching *_workspace_size */
  MLA_ERR_CUDA = 4,          /* a CUDA runtime call failed (launch error, bad device) */
  MLA_ERR_TIMEOUT = 5,       /* device: a bounded wait inside a kernel gave up */
  MLA_ERR_DEVICE_CHECK = 6   /* device: an index read from device memory was out of range */
};

enum mla_dtype { MLA_F32 = 0, MLA_BF16 = 1 };

/* Shapes of one layer. sm_scale multiplies every score; 0 selects 1/sqrt(D + d_r), the scale of
 * « L'obstacle : RoPE » (a negative or NaN value is an invalid argument). */
typedef struct mla_dims {
  int32_t H;          /* query heads */
  int32_t D;          /* no-RoPE width of a query/key head (qk_nope) */
  int32_t d_r;        /* width of the decoupled RoPE key, shared by all heads; even */
  int32_t d_c;        /* latent width */
  int32_t d_v;        /* value head width */
  int32_t g;          /* GQLA groups, H % g == 0 (0 when the grouped path is not used) */
  int32_t page_size;  /* positions per cache page; must be 64 */
  float sm_scale;     /* score scale; 0 = 1/sqrt(D + d_r) */
  float rms_eps;      /* RMSNorm epsilon: c = z / sqrt(mean(z^2) + rms_eps) * gamma */
  float rope_base;    /* RoPE: pair (2i, 2i+1) turns by pos * rope_base^(-2i/d_r) */
} mla_dims_t;

/* Latent cache pool: latent rows [num_pages*64, d_c] and RoPE-key rows [num_pages*64, d_r].
 * The two may be one interleaved array (rope = latent + d_c, both strides d_c + d_r). */
typedef struct mla_latent_cache {
  void* latent;           /* device, dtype */
  int64_t latent_stride;  /* elements from one row to the next, >= d_c */
  void* rope;             /* device, dtype */
  int64_t rope_stride;    /* elements from one row to the next, >= d_r */
  int32_t num_pages;      /* pages in the pool; page ids must be < num_pages */
} mla_latent_cache_t;

/* Expanded GQA cache of the grouped path (« Chemin GQA »): per row, keys [g, D], values
 * [g, d_v] and the shared RoPE key [d_r]. */
typedef struct mla_gqa_cache {
  void* k;  int64_t k_stride;     /* [num_pages*64, g, D]; stride = elements between rows */
  void* v;  int64_t v_stride;     /* [num_pages*64, g, d_v] */
  void* rope; int64_t rope_stride;/* [num_pages*64, d_r] */
  int32_t num_pages;
} mla_gqa_cache_t;

/* ---------------------------------------------------------------------------------------------
 * a1. Cache append (« L'idée : garder un résumé »; « L'obstacle : RoPE »).
 * For each new token (b, t): z = x[b,t,:] · W where W = [W_DKV | W_KR] is [C, d_c + d_r];
 *   c   = z[0:d_c] / sqrt(mean(z[0:d_c]^2) + rms_eps) * gamma      (gamma NULL means all ones)
 *   k_r = RoPE(z[d_c:d_c+d_r], position)
 * and writes c and k_r into the cache row of that token's position.
 *   x       [B, s_q, C] dtype          w_dkv_kr [C, d_c + d_r] dtype      gamma [d_c] dtype or NULL
 *   seqlens [B] int32                   block_table [B, max_pages] int32
 * workspace: at least mla_append_workspace_size(...) bytes of device memory (fp32 partial sums);
 * its contents need not be initialised.
 * ------------------------------------------------------------------------------------------- */
MLA_API size_t mla_append_workspace_size(const mla_dims_t* dims, int32_t B, int32_t s_q, int32_t C);
MLA_API int mla_append_cache(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q,
                     const void* x, int32_t C, const void* w_dkv_kr, const void* gamma,
                     const int32_t* seqlens, const int32_t* block_table, int32_t max_pages,
                     const mla_latent_cache_t* cache, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------------
 * a1 without a workspace. The pages have no counterpart to this call: it exists for callers that
 * cannot allocate device memory — code running inside a framework whose memory pool owns the
 * device and forbids side allocations, plugins that only receive the tensors of the call, or a
 * serving process that must not call cudaMalloc once it is running. Same arguments and result as
 * mla_append_cache, minus the workspace: the split-K partial sums go to a 4 MiB buffer that is
 * part of the library's device image (every GPU that loads the library holds it until exit).
 * Nothing is allocated or freed. Limit: B * s_q * (d_c + d_r) <= 1,048,576, else
 * MLA_ERR_WORKSPACE is returned and nothing is launched. In bf16 with C a multiple of 64 the
 * projection runs on the tensor cores, as in mla_append_cache. The first call on each device looks
 * up the buffer's device address (with that device current) and caches it; make that first call
 * before any stream capture. A reset of the device (cudaDeviceReset) makes the cached address
 * stale: after one, this call must not be used again in the same process. All calls share the
 * buffer: calls that overlap on the GPU (streams with no ordering between them) race on it.
 * Nothing in it needs to start at zero.
 * ------------------------------------------------------------------------------------------- */
MLA_API int mla_append_cache_noalloc(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q,
                             const void* x, int32_t C, const void* w_dkv_kr, const void* gamma,
                             const int32_t* seqlens, const int32_t* block_table, int32_t max_pages,
                             const mla_latent_cache_t* cache, void* stream);

/* ---------------------------------------------------------------------------------------------
 * f2. Query projection chain (« L'attention latente … », « L'obstacle : RoPE » and « Le code »:
 * the query of a new token also passes through a low-rank latent, normalised like the cache's):
 *   c_q        = RMSNorm(x[b,t,:] · W_DQ) · gamma_q          (width d_q; eps = dims->rms_eps)
 *   q_nope     = c_q · W_UQ, split into H heads of D          -> q_nope [B, s_q, H, D]
 *   q_rope_raw = c_q · W_QR, split into H heads of d_r        -> q_rope_raw [B, s_q, H, d_r]
 * q_rope_raw is not rotated: mla_absorb_q rotates it at the token's position. c_q is rounded to
 * dtype once, between the two projections (as the cache's latent rows are).
 *   x [B, s_q, C]   w_dq [C, d_q]   gamma_q [d_q] or NULL (= 1)   w_uq [d_q, H*D]   w_qr [d_q, H*d_r]
 *   (all dtype, row-major, 16-byte aligned)
 * workspace: at least mla_query_workspace_size(...) bytes of device memory (fp32 partial sums of
 * x·W_DQ, then c_q); its contents need not be initialised. Errors: MLA_ERR_INVALID_ARG for null or
 * misaligned pointers and non-positive sizes, MLA_ERR_WORKSPACE, MLA_ERR_CUDA (see the conventions
 * above: the chain enqueues three or four kernels).
 * ------------------------------------------------------------------------------------------- */
MLA_API size_t mla_query_workspace_size(const mla_dims_t* dims, int32_t B, int32_t s_q, int32_t C, int32_t d_q);
MLA_API int mla_project_query(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q,
                      const void* x, int32_t C, int32_t d_q, const void* w_dq, const void* gamma_q,
                      const void* w_uq, const void* w_qr, void* q_nope, void* q_rope_raw,
                      void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------------
 * a2. Query absorption (« Ce que DeepSeek fait de plus »: q·(W_UK c) = (q·W_UK)·c).
 *   q_abs[b,t,h, 0:d_c]       = q_nope[b,t,h,:] · W_UK[h]            (W_UK[h] is [D, d_c])
 *   q_abs[b,t,h, d_c:d_c+d_r] = RoPE(q_rope_raw[b,t,h,:], seqlens[b] - s_q + t)
 *   q_nope [B, s_q, H, D]   q_rope_raw [B, s_q, H, d_r]   w_uk [H, D, d_c]   seqlens [B] int32
 *   q_abs  [B, s_q, H, d_c + d_r]   (all dtype)
 * ------------------------------------------------------------------------------------------- */
MLA_API int mla_absorb_q(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q,
                 const void* q_nope, const void* q_rope_raw, const void* w_uk,
                 const int32_t* seqlens, void* q_abs, void* stream);

/* ---------------------------------------------------------------------------------------------
 * a1 and a2 of one decode step in one call: mla_append_cache, then mla_absorb_q, on one stream.
 * The order is the one that overlaps best: the absorption's CTAs (one per head) stream W_UK while
 * the append's finish (RMSNorm, RoPE, paged store) runs. Arguments, layouts and results are those of
 * the two calls, bit for bit. workspace: at least mla_append_workspace_size(dims, B, s_q, C) bytes,
 * no initialisation needed. Argument errors of either half return before anything is launched.
 * Weights (w_dkv_kr, w_uk here, w_uv and w_o in mla_out_proj) may be read before the kernel
 * launched just before on the stream has finished, when that kernel lets its successor start early
 * (programmatic dependent launch): such a kernel must not write them. No kernel of this library
 * writes an array that one of these calls takes as a weight.
 * ------------------------------------------------------------------------------------------- */
MLA_API int mla_append_cache_absorb_q(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q,
                              const void* x, int32_t C, const void* w_dkv_kr, const void* gamma,
                              const void* q_nope, const void* q_rope_raw, const void* w_uk,
                              const int32_t* seqlens, const int32_t* block_table, int32_t max_pages,
                              const mla_latent_cache_t* cache, void* q_abs, void* workspace,
                              size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------------
 * a3 + a4. Absorbed decode over the latent cache, split over the GPU's SMs, with the
 * log-sum-exp merge of split sequences (« Chemin MQA-Absorbé »; « Le mécanisme d'attention »).
 * For each (b, t, h), over the visible positions j:
 *   s_j   = sm_scale * (q_abs[b,t,h,0:d_c] · c_j + q_abs[b,t,h,d_c:] · k_r,j)
 *   o_lat[b,t,h,:] = sum_j softmax(s)_j * c_j          lse[b,t,h] = log sum_j exp(s_j)
 *   q_abs [B, s_q, H, d_c + d_r] dtype    o_lat [B, s_q, H, d_c] dtype    lse [B, s_q, H] fp32
 * workspace: at least mla_decode_workspace_size(...) bytes (split partials); no initialisation
 * needed. The size depends on the current device's SM count and on max_pages (the longest
 * sequence the table can describe is max_pages*64 positions).
 * Requires every seqlens[b] >= s_q (a token always sees itself).
 * ------------------------------------------------------------------------------------------- */
MLA_API size_t mla_decode_workspace_size(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q,
                                 int32_t max_pages);
MLA_API int mla_decode_absorbed(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q,
                        const void* q_abs, const mla_latent_cache_t* cache,
                        const int32_t* block_table, int32_t max_pages, const int32_t* seqlens,
                        void* o_lat, float* lse, void* workspace, size_t ws_bytes, void* stream);
/* The same call given a host copy of the lengths (seqlens_host: B int32 in host memory, equal to
 * seqlens; NULL is mla_decode_absorbed). The tensor-core decode cuts sequences between its worker
 * pairs only when the batch is unbalanced; the copy lets the host see beforehand that nothing will
 * be cut, and the decode then goes as one plain launch without the split merge machinery (at the
 * bench shape a few microseconds less per call). If the device's seqlens nevertheless make the
 * kernel cut a sequence (the copy was stale), that sequence's outputs are left unmerged and
 * MLA_ERR_DEVICE_CHECK is recorded. The copy is read during the call only. */
MLA_API int mla_decode_absorbed_hinted(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q,
                               const void* q_abs, const mla_latent_cache_t* cache,
                               const int32_t* block_table, int32_t max_pages, const int32_t* seqlens,
                               const int32_t* seqlens_host, void* o_lat, float* lse, void* workspace,
                               size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------------
 * a5. Output projection (« Ce que DeepSeek fait de plus »: the weighted latent sum is projected
 * once by W_UV; « Le code »: the layer's final projection).
 *   out[b,t,h,:] = o_lat[b,t,h,:] · W_UV[h]                   (W_UV[h] is [d_c, d_v])
 *   if w_o != NULL: out_model[b,t,:] = concat_h(out[b,t,h,:]) · W_O   (W_O is [H*d_v, C]; in bf16 with
 *   H*d_v a multiple of 64 and C of 8 this second product runs on the tensor cores too)
 *   o_lat [B, s_q, H, d_c]  w_uv [H, d_c, d_v]  out [B, s_q, H, d_v]  out_model [B, s_q, C] (dtype)
 * ------------------------------------------------------------------------------------------- */
MLA_API int mla_out_proj(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q,
                 const void* o_lat, const void* w_uv, void* out,
                 const void* w_o, int32_t C, void* out_model, void* stream);

/* ---------------------------------------------------------------------------------------------
 * a6. GQLA grouped decode (« Résumé technique : GQLA … », « Architecture » and « Chemin GQA »).
 * Head h uses group h / (H/g). For each (b, t, h) over the visible positions j:
 *   s_j = sm_scale * (q_nope[b,t,h,:] · K[j, g(h), :] + RoPE(q_rope_raw[b,t,h,:], pos_t) · k_r,j)
 *   out[b,t,h,:] = sum_j softmax(s)_j * V[j, g(h), :]          lse[b,t,h] = log sum_j exp(s_j)
 *   q_nope [B, s_q, H, D]  q_rope_raw [B, s_q, H, d_r]  out [B, s_q, H, d_v] (dtype)  lse fp32
 * workspace: at least mla_gqla_workspace_size(...) bytes.
 * Requires every seqlens[b] >= s_q, as a3 does: a sequence shorter than that is reported on the
 * device (MLA_ERR_DEVICE_CHECK) and its outputs are undefined.
 * ------------------------------------------------------------------------------------------- */
MLA_API size_t mla_gqla_workspace_size(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q,
                               int32_t max_pages);
MLA_API int mla_decode_gqla_grouped(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q,
                            const void* q_nope, const void* q_rope_raw, const mla_gqa_cache_t* cache,
                            const int32_t* block_table, int32_t max_pages, const int32_t* seqlens,
                            void* out, float* lse, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------------
 * f3. Append to the expanded GQA cache of the grouped path (« Résumé technique : GQLA … »,
 * « Chemin GQA »: the latent is expanded into g key/value groups once, when the cache is written).
 * For each new token (b, t) at position seqlens[b] - s_q + t:
 *   c   = RMSNorm(x[b,t,:] · W_DKV) · gamma            (rounded to dtype, as a latent cache row is)
 *   k_r = RoPE(x[b,t,:] · W_KR, position)             -> cache->rope row
 *   K[g] = W_UK[g] · c   (W_UK [g, D, d_c])           -> cache->k row [g, D]
 *   V[g] = c · W_UV[g]   (W_UV [g, d_c, d_v])         -> cache->v row [g, d_v]
 *   x [B, s_q, C]   w_dkv_kr [C, d_c + d_r]   gamma [d_c] or NULL   (all dtype)
 * Only MLA_BF16 with C and d_c multiples of 64 and D, d_v multiples of 8 (else MLA_ERR_UNSUPPORTED).
 * workspace: at least mla_gqa_append_workspace_size(...) bytes (fp32 partial sums, then c, K and V of
 * the new tokens); contents need not be initialised. The call enqueues five kernels.
 * ------------------------------------------------------------------------------------------- */
MLA_API size_t mla_gqa_append_workspace_size(const mla_dims_t* dims, int32_t B, int32_t s_q, int32_t C);
MLA_API int mla_append_gqa_cache(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q, const void* x, int32_t C,
                         const void* w_dkv_kr, const void* gamma, const void* w_uk_g, const void* w_uv_g,
                         const int32_t* seqlens, const int32_t* block_table, int32_t max_pages,
                         const mla_gqa_cache_t* cache, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------------
 * f3. The value up-projection absorbed into the output projection (« Résumé technique : GQLA … »,
 * « Chemin MQA-Absorbé »: the up-projections are absorbed into the query and output projections).
 * mla_preabsorb_out_weights builds, once per layer, W_UVO[h] = W_UV[h] · W_O[h*d_v : (h+1)*d_v, :]:
 *   w_uv [H, d_c, d_v]   w_o [H*d_v, C]   ->   w_uvo [H, d_c, C]   (all dtype; H GEMMs enqueued)
 * mla_out_proj_preabsorbed then computes the layer output straight from the weighted latents:
 *   out_model[b,t,:] = concat_h(o_lat[b,t,h,:]) · W_UVO     (o_lat [B, s_q, H, d_c], w_uvo as above)
 * which equals mla_out_proj with w_o up to rounding. Note the weight is H*d_c x C: it pays off only
 * when d_c * H * C is small against the two projections it replaces.
 * ------------------------------------------------------------------------------------------- */
MLA_API int mla_preabsorb_out_weights(const mla_dims_t* dims, int32_t dtype, const void* w_uv, const void* w_o, int32_t C,
                              void* w_uvo, void* stream);
MLA_API int mla_out_proj_preabsorbed(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q, const void* o_lat,
                             const void* w_uvo, int32_t C, void* out_model, void* stream);

/* ---------------------------------------------------------------------------------------------
 * 8-bit latent cache (« Cache KV, mémoire récurrente, MLA et bas rang », trainer notes of « Le
 * problème — Cache KV standard »: one byte per cached value instead of two). Only the latent rows
 * are narrowed; the RoPE keys stay in dtype. Each latent row j is stored as FP8 E4M3 codes (1 sign,
 * 4 exponent bits of bias 7, 3 mantissa bits, subnormals, largest finite value 448) with one fp32
 * scale s_j = max|c_j| / 448:
 *   code_j = E4M3(c_j / s_j), round to nearest, ties to even, saturated at +-448 (s_j and the
 *   quotients computed in fp32, each rounded once); a zero row stores s_j = 0 and zero codes.
 * The decode attends the dequantised rows s_j * value(code_j) exactly as mla_decode_absorbed attends
 * 16-bit rows (same q_abs, o_lat, lse, seqlens and table conventions).
 *
 * mla_quantize_latent_fp8: rows [0, rows) of `latent` (dtype, row stride `latent_stride` elements,
 *   >= d_c) into codes [rows, d_c] (uint8, row stride `code_stride` bytes, >= d_c, multiple of 16)
 *   and scales [rows] (fp32). Any row range of a pool can be converted (for example the rows that
 *   mla_append_cache has just written, or a whole 16-bit pool once). Errors: MLA_ERR_INVALID_ARG
 *   (null or misaligned pointers, bad strides, rows <= 0), MLA_ERR_UNSUPPORTED (d_c not a multiple
 *   of 16).
 * mla_decode_absorbed_fp8: a3 + a4 over that cache. The cache descriptor names the codes, the
 *   scales and the dtype RoPE keys of the same num_pages*64 rows. workspace: at least
 *   mla_decode_fp8_workspace_size(...) bytes, no initialisation needed. In bf16 at the shapes of
 *   the tensor-core decode (H = 128, d_c = 512, d_r = 64, s_q <= 8) the pages the batch reads are
 *   first dequantised into the workspace (bf16 rows s * value(code), rounded once, and the RoPE keys:
 *   B * max_pages * 64 * (d_c + d_r) * 2 bytes, plus a dense page table and the decode's own
 *   workspace), and the tensor-core decode runs over them; otherwise the decode runs on the CUDA
 *   cores (fp32 arithmetic). Requires every seqlens[b] >= s_q. Same errors as mla_decode_absorbed.
 * ------------------------------------------------------------------------------------------- */
typedef struct mla_latent_cache_fp8 {
  const uint8_t* codes;   /* device, [num_pages*64, >= d_c] E4M3 codes of the latent rows */
  int64_t code_stride;    /* bytes from one row of codes to the next, >= d_c, multiple of 16 */
  const float* scales;    /* device, [num_pages*64] one fp32 scale per row */
  const void* rope;       /* device, dtype, [num_pages*64, >= d_r] RoPE keys */
  int64_t rope_stride;    /* elements from one RoPE row to the next, >= d_r */
  int32_t num_pages;      /* pages in the pool; page ids must be < num_pages */
} mla_latent_cache_fp8_t;

MLA_API int mla_quantize_latent_fp8(const mla_dims_t* dims, int32_t dtype, const void* latent, int64_t latent_stride,
                                    int64_t rows, uint8_t* codes, int64_t code_stride, float* scales, void* stream);
MLA_API size_t mla_decode_fp8_workspace_size(const mla_dims_t* dims, int32_t B, int32_t s_q, int32_t max_pages);
MLA_API int mla_decode_absorbed_fp8(const mla_dims_t* dims, int32_t dtype, int32_t B, int32_t s_q, const void* q_abs,
                                    const mla_latent_cache_fp8_t* cache, const int32_t* block_table,
                                    int32_t max_pages, const int32_t* seqlens, void* o_lat, float* lse,
                                    void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------------
 * Status.
 * mla_check_status: synchronises `stream`, returns the device status word of the current device
 * (MLA_OK when no kernel recorded an error since the last call) and clears it.
 * mla_status_string: a static, human-readable name of a status code.
 * mla_build_info: a static string naming the build (target architecture, kernels compiled in).
 * mla_launch_count: kernels this process has launched through the library so far (host counter,
 * incremented at every launch; used to report how many kernels a timed region ran).
 * ------------------------------------------------------------------------------------------- */
MLA_API int mla_check_status(void* stream);
MLA_API const char* mla_status_string(int status);
MLA_API const char* mla_build_info(void);
MLA_API uint64_t mla_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* MLA_H_ */
