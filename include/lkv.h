/*
 * lkv.h -- C ABI of the B200 (sm_100a) latent / grouped KV-cache decode-attention library.
 *
 * One decode step for a batch of requests: every request b has a contiguous run of
 * L_b cached tokens starting at row cu_seqlens[b] of the cache arrays; its s_q (1 or 2)
 * newest tokens are already the last s_q rows of that run.  Query token i of request b
 * attends to rows 0 .. L_b - s_q + i of its run (causal inside the new tokens).  For query
 * head h of group j = h / (h_q / G):
 *
 *   s[t]  = scale * ( q[b,i,h,:] . K_j[t,:]  +  q_rope[b,i,h,:] . k_rope[t,:] )
 *   lse   = ln sum_t exp(s[t])
 *   out   = sum_t exp(s[t] - lse) * V_j[t,:]
 *
 * Forms (sources: "GQLA: Group-Query Latent Attention for Hardware-Adaptive Large Language
 * Model Decoding", section 2 "Methodology"; "Grouped Latent Attention" article, section "GLA"):
 *   - MLA absorbed path (section 2, "MQA absorbed path"): G = 1, K = V = the latent c_KV
 *     (width r_kv), plus one RoPE key of width d_R shared by all heads.  The query carries
 *     W_UK already (q_nope_abs); the output is in latent space.
 *   - GQLA GQA path (section 2, "GQA path"): the latent expanded once into g groups of
 *     keys K_j and values V_j (width d_h each) plus the shared RoPE key.
 *   - GLA: n_lat latent groups of width r_g; group j's heads use latent group j as both
 *     K_j and V_j; one RoPE key shared by all groups.
 *
 * Conventions for every entry point:
 *   - All pointers are device pointers unless stated; the caller allocates every buffer,
 *     including the workspace.  The library allocates no device memory in these calls.
 *   - Calls are asynchronous on `stream` (cudaStream_t; NULL = legacy default stream).
 *   - Argument errors are detected on the host before anything is launched and returned
 *     as LKV_ERR_INVALID_ARG / LKV_ERR_UNSUPPORTED / LKV_ERR_WORKSPACE.  These checks make
 *     no CUDA call.
 *   - Faults found on the device (a bounded wait that gave up, a cache length below s_q,
 *     a destination row past the cache) never trap: the kernel records a site code in a
 *     device error word, skips the bad access and unwinds.  lkv_check_device() reads it.
 *   - "bf16" means bf16 storage with fp32 accumulation; lse is always fp32, natural log.
 *   - scale must be finite and > 0 (the pages' softmax scale is 1/sqrt of the score width);
 *     a positive scale keeps the order of the raw scores, which the kernels rely on.
 *   - Row strides are in elements and must keep every row 16-byte aligned.
 *   - The first call on a device sets that device up for the rest of the process (SM count,
 *     kernel attributes, device addresses of the library's own device variables).  After a
 *     cudaDeviceReset of a device the library must not be called on that device again in the
 *     same process: the kept addresses would point into the released context.
 */
#ifndef LKV_H
#define LKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* lkv_stream_t; /* same type as cudaStream_t */

typedef enum {
  LKV_OK = 0,
  LKV_ERR_INVALID_ARG = 1, /* null pointer, bad size, stride or alignment; nothing launched */
  LKV_ERR_UNSUPPORTED = 2, /* well formed but outside the implemented shapes / dtypes */
  LKV_ERR_WORKSPACE = 3,   /* workspace null or smaller than the *_workspace_size value */
  LKV_ERR_CUDA = 4,        /* a CUDA runtime call failed (launch, attribute, tensor map) */
  LKV_ERR_DEVICE = 5       /* lkv_check_device: a kernel recorded a device-side failure */
} lkv_status;

typedef enum { LKV_BF16 = 0, LKV_FP32 = 1 } lkv_dtype;

/* Library version (major*10000 + minor*100 + patch). */
int lkv_version(void);

/* Static description of a status code.  Never NULL. */
const char* lkv_status_string(int status);

/*
 * Work partition used by the decode kernels (host-only, no CUDA call).  The tiles of all
 * (request, unit) pairs are laid end to end and cut into `ranges` equal runs, one per
 * persistent CTA (MLA: per CTA pair).  A unit is one query token of a request for MLA,
 * one group of a request for GQLA / GLA.  Returns the number of ranges, or -1 on bad input.
 *   kind: 0 = MLA absorbed, 1 = GQLA, 2 = GLA, 3 = GTA (partitioned like GQLA), 4 = GLA whose
 *   units have at most 64 rows (s_q * h_q / groups <= 64: the ranges of kind 2).
 *   num_sms: SMs available on the device.
 */
int lkv_plan_ranges(int kind, int batch, int s_q, int groups, int num_sms);

/*
 * Host-only view of the same partition (no CUDA call): for host-side cu_seqlens_host [batch+1]
 * and `num_ranges` ranges, writes one record of 8 int32 per segment, in processing order:
 *   (range, request, unit, tile_lo, tile_hi, complete, slot, unit_id)
 * tiles are 256 keys (MLA), 128 keys (GQLA, GTA, GLA units of at most 64 rows: kind 4) or 64 keys
 * (GLA units of more rows: kind 2); slot is -1 for a segment that covers its whole unit, else the partial
 * slot (0 = first segment of its range, 1 = last).  Returns the number of segments (records
 * past max_out are counted but not written), or -1 on bad input.
 */
int lkv_plan_segments(int kind, const int32_t* cu_seqlens_host, int batch, int s_q, int groups,
                      int num_ranges, int32_t* out, int max_out);

/* Bytes of workspace the decode entry points need (host-only, no CUDA call); 0 on bad input.
 * The workspace holds fp32 partial outputs / LSEs for units that straddle a range boundary
 * and the record of which unit each partial belongs to.  Its contents need no initialisation
 * and are fully rewritten by every call. */
size_t lkv_mla_decode_workspace_size(int batch, int s_q, int h_q, int r_kv, int num_sms);
size_t lkv_group_decode_workspace_size(int kind, int batch, int s_q, int h_q, int groups,
                                       int d_v, int num_sms);

/*
 * MLA absorbed decode (MQA over the shared latent).
 *   q_nope_abs [batch, s_q, h_q, r_kv]  contiguous, query with W_UK folded in
 *   q_rope     [batch, s_q, h_q, d_rope] contiguous
 *   ckv        [cache_rows, r_kv]  row stride ckv_row_stride (elements)
 *   kpe        [cache_rows, d_rope] row stride kpe_row_stride (ckv and kpe may interleave in
 *              one [cache_rows, r_kv + d_rope] array: kpe = ckv + r_kv, same stride)
 *   cu_seqlens [batch + 1] int32, device; cu_seqlens[batch] <= cache_rows;
 *              every L_b = cu_seqlens[b+1] - cu_seqlens[b] >= s_q (checked on the device: a shorter
 *              request is recorded as LKV_SITE_BAD_LENGTH and its outputs are not written)
 *   out        [batch, s_q, h_q, r_kv] (bf16 for LKV_BF16, fp32 for LKV_FP32)
 *   lse        [batch, s_q, h_q] fp32
 * Implemented: LKV_BF16 with r_kv = 512, d_rope = 64, h_q = 128 (tcgen05 kernel on CTA pairs that
 *              share one MMA, 256-key tiles);
 *              LKV_FP32 with r_kv + d_rope <= 1024, r_kv <= 512 (CUDA-core kernel).
 * s_q must be 1 or 2.  workspace_bytes >= lkv_mla_decode_workspace_size(...).
 */
lkv_status lkv_mla_absorbed_decode(const void* q_nope_abs, const void* q_rope, const void* ckv,
                                   int64_t ckv_row_stride, const void* kpe,
                                   int64_t kpe_row_stride, int64_t cache_rows,
                                   const int32_t* cu_seqlens, int batch, int s_q, int h_q,
                                   int r_kv, int d_rope, float scale, int dtype, void* out,
                                   float* lse, void* workspace, size_t workspace_bytes,
                                   lkv_stream_t stream);

/*
 * GQLA grouped decode (GQA path over g expanded key/value groups).
 *   q      [batch, s_q, h_q, d_h], q_rope [batch, s_q, h_q, d_rope] contiguous
 *   k, v   [cache_rows, g, d_h] with row strides k_row_stride / v_row_stride (elements per
 *          cache row, >= g*d_h); kpe [cache_rows, d_rope] row stride kpe_row_stride
 *   out    [batch, s_q, h_q, d_h]; lse [batch, s_q, h_q]
 * Implemented: LKV_BF16 with d_h = 128, d_rope = 64, h_q / g <= 64, s_q * h_q / g <= 128;
 *              LKV_FP32 with d_h + d_rope <= 1024, d_h <= 512.
 */
lkv_status lkv_gqla_group_decode(const void* q, const void* q_rope, const void* k,
                                 int64_t k_row_stride, const void* v, int64_t v_row_stride,
                                 const void* kpe, int64_t kpe_row_stride, int64_t cache_rows,
                                 const int32_t* cu_seqlens, int batch, int s_q, int h_q, int g,
                                 int d_h, int d_rope, float scale, int dtype, void* out,
                                 float* lse, void* workspace, size_t workspace_bytes,
                                 lkv_stream_t stream);

/*
 * GLA grouped-latent decode.
 *   q      [batch, s_q, h_q, r_g], q_rope [batch, s_q, h_q, d_rope] contiguous
 *   clat   [cache_rows, n_lat * r_g] row stride clat_row_stride; group j = columns
 *          j*r_g .. (j+1)*r_g - 1; kpe [cache_rows, d_rope] row stride kpe_row_stride
 *   out    [batch, s_q, h_q, r_g]; lse [batch, s_q, h_q]
 * Implemented: LKV_BF16 with r_g = 256, d_rope = 64, s_q * h_q / n_lat <= 128;
 *              LKV_FP32 with r_g + d_rope <= 1024, r_g <= 512.
 */
lkv_status lkv_gla_group_decode(const void* q, const void* q_rope, const void* clat,
                                int64_t clat_row_stride, const void* kpe, int64_t kpe_row_stride,
                                int64_t cache_rows, const int32_t* cu_seqlens, int batch, int s_q,
                                int h_q, int n_lat, int r_g, int d_rope, float scale, int dtype,
                                void* out, float* lse, void* workspace, size_t workspace_bytes,
                                lkv_stream_t stream);

/*
 * GTA (grouped-tied attention) decode: the heads of group j read one tied state per cached token
 * as both their key (with the shared RoPE key appended) and their value.  Source: the Grouped
 * Latent Attention article (news page), section "GTA": K and V parameters are tied inside a
 * group, so the cache holds g*d_h + d_rope elements per token, about half of GQA's.
 *   q      [batch, s_q, h_q, d_h], q_rope [batch, s_q, h_q, d_rope] contiguous
 *   kv     [cache_rows, g, d_h] row stride kv_row_stride (elements, >= g*d_h); kpe
 *          [cache_rows, d_rope] row stride kpe_row_stride (kv and kpe may interleave in one
 *          [cache_rows, g*d_h + d_rope] array)
 *   out    [batch, s_q, h_q, d_h]; lse [batch, s_q, h_q]
 * Runs the grouped tensor-core kernel in its tied mode: each tile of tied states (with the RoPE
 * key) is read once into shared memory and serves as the key operand of QK and the value operand
 * of PV.  Same limits as lkv_gqla_group_decode, same workspace (lkv_group_decode_workspace_size
 * with kind 1 or 3).
 */
lkv_status lkv_gta_group_decode(const void* q, const void* q_rope, const void* kv,
                                int64_t kv_row_stride, const void* kpe, int64_t kpe_row_stride,
                                int64_t cache_rows, const int32_t* cu_seqlens, int batch, int s_q,
                                int h_q, int g, int d_h, int d_rope, float scale, int dtype,
                                void* out, float* lse, void* workspace, size_t workspace_bytes,
                                lkv_stream_t stream);

/*
 * GTA decode over FP8 cache rows (the row format of lkv_fp8_cache_row_bytes below, with
 * r = g * d_h): the tied state of group j is the dequantised columns [128 j, 128 j + 128) of the
 * row's latent, e4m3(code) * s, used as key (with the row's bf16 RoPE key) and as value, exactly as
 * lkv_gta_group_decode uses its bf16 tied rows.  FP8 halves the bytes of the tied states (the pages
 * run their latent models in FP8 for serving: Grouped Latent Attention article, section on the
 * GLA-vs-MLA decoding test).
 *   cache  [cache_rows] FP8 rows of cache_row_stride_bytes (a multiple of 16), 16-byte aligned
 *   q, q_rope, cu_seqlens, out, lse, workspace: as lkv_gta_group_decode (bf16); the workspace size
 *          is lkv_group_decode_workspace_size with kind 3.
 * Implemented: d_h = 128, d_rope = 64, g * d_h <= 1024, s_q * h_q / g <= 64 (LKV_ERR_UNSUPPORTED
 * otherwise).  Rows past a unit's keys are never read as values (their codes are not converted).
 */
lkv_status lkv_gta_group_decode_fp8(const void* q, const void* q_rope, const void* cache,
                                    int64_t cache_row_stride_bytes, int64_t cache_rows,
                                    const int32_t* cu_seqlens, int batch, int s_q, int h_q, int g, int d_h,
                                    int d_rope, float scale, void* out, float* lse, void* workspace,
                                    size_t workspace_bytes, lkv_stream_t stream);

/*
 * GQLA grouped decode that allocates nothing and takes no workspace.
 *
 * No counterpart on the source pages.  It serves callers that cannot allocate device memory
 * on the decode path: hosts without a device allocator of their own, and serving loops that
 * reserve all device memory up front and must not call cudaMalloc (which may also synchronise
 * the device) per step.  Arguments and results are those of lkv_gqla_group_decode without the
 * workspace.  The split-KV partials go to one fixed device array inside the library of
 * LKV_STATIC_SCRATCH_BYTES (8 MiB), which every GPU that loads the library keeps until the
 * process exits.
 *   - A shape whose workspace (lkv_group_decode_workspace_size) exceeds that size is rejected
 *     with LKV_ERR_WORKSPACE before anything is launched.
 *   - All calls on a device share the array and it keeps the last call's contents.  The kernel
 *     writes everything it later reads, so nothing needs clearing, but two calls that overlap
 *     on the GPU (e.g. unordered streams) race on it.
 *   - The first call on a device looks up the array's device address with that device
 *     current; make that first call before any stream capture begins.
 *   - It calls no cudaMalloc, no cudaFree and no allocating library routine.
 */
#define LKV_STATIC_SCRATCH_BYTES (8u << 20)
lkv_status lkv_gqla_group_decode_noalloc(const void* q, const void* q_rope, const void* k,
                                         int64_t k_row_stride, const void* v,
                                         int64_t v_row_stride, const void* kpe,
                                         int64_t kpe_row_stride, int64_t cache_rows,
                                         const int32_t* cu_seqlens, int batch, int s_q, int h_q,
                                         int g, int d_h, int d_rope, float scale, int dtype,
                                         void* out, float* lse, lkv_stream_t stream);

/*
 * Cache append: copy the s_q new rows of every request into the cache.
 * Row b*s_q + i of new_rows goes to cache row cu_seqlens[b] + L_b - s_q + i (the new tokens
 * are the tail of each request's run; source: GQLA explainer, section 2 -- the cache holds
 * the latent and RoPE key per token, or the expanded groups on the GQA path).
 *   new_rows  [batch*s_q rows] of row_bytes each, row stride new_row_stride_bytes
 *   cache     [cache_rows rows], row stride cache_row_stride_bytes
 * row_bytes, both strides and both pointers must be multiples of 16.  A request with
 * L_b < s_q or a destination past cache_rows is skipped and recorded in the device error word.
 */
lkv_status lkv_latent_cache_append(const void* new_rows, int64_t new_row_stride_bytes,
                                   void* cache, int64_t cache_row_stride_bytes,
                                   int64_t cache_rows, int64_t row_bytes,
                                   const int32_t* cu_seqlens, int batch, int s_q,
                                   lkv_stream_t stream);

/*
 * Output projection y = o W_O (bf16 operands, fp32 accumulation; the tensor-core GEMM of the other
 * projections).
 *   o    [n_tok, k] bf16 row-major: the heads' attention outputs side by side (k = heads * d_v)
 *   w_o  [k, d_model] bf16 row-major
 *   y    [n_tok, d_model], bf16 (out_dtype LKV_BF16) or fp32 (LKV_FP32)
 * With the heads split along the group axis across GPUs (GQLA explainer, section 2, GQA path), each
 * GPU passes its heads' columns of o and the matching row block of W_O and gets a partial y; the sum
 * over GPUs is the full projection.  LKV_ERR_INVALID_ARG for NULL pointers, non-positive sizes,
 * another out_dtype, o or w_o not 16-byte aligned, or k or d_model not a multiple of 8.
 */
lkv_status lkv_output_projection(const void* o, const void* w_o, void* y, int n_tok, int k, int d_model,
                                 int out_dtype, lkv_stream_t stream);

/*
 * FP8 (e4m3) latent cache rows (the pages run FP8 inference -- Grouped Latent Attention article,
 * section on the GLA-vs-MLA decoding test -- but fix no format; this is the library's reading).
 * One row per token of lkv_fp8_cache_row_bytes(r, d_rope) = r + 16 + 2*d_rope bytes:
 *   bytes [0, r)          e4m3 codes of the latent row (OCP E4M3: bias 7, largest finite 448)
 *   bytes [r, r + 4)      fp32 scale s: the smallest power of two with max|latent row| / s <= 448
 *                         (0 for an all-zero row)
 *   bytes [r + 4, r + 16) zero
 *   bytes [r + 16, ...)   the bf16 RoPE key, copied unchanged
 * The dequantised latent is e4m3(code) * s, exact in bf16 (a power of two times a 4-bit
 * significand).  Codes: y = x / s (exact), rounded to the nearest e4m3 value with ties to the even
 * code.
 * lkv_fp8_cache_row_bytes returns 0 unless r is a multiple of 16 in [16, 1024] and d_rope a
 * non-negative multiple of 8 (host-only, no CUDA call).
 */
size_t lkv_fp8_cache_row_bytes(int r, int d_rope);

/*
 * Quantise n_rows bf16 rows into FP8 cache rows, row i to row i.
 *   src    [n_rows, >= r + d_rope] bf16: latent in columns [0, r), RoPE key in [r, r + d_rope);
 *          row stride src_row_stride elements (its byte size a multiple of 16); 16-byte aligned
 *   cache  [n_rows] rows of cache_row_stride_bytes (a multiple of 16, >= the row size), aligned
 * Source values must be finite.  Asynchronous on `stream`.
 */
lkv_status lkv_quantize_latent_fp8(const void* src, int64_t src_row_stride, void* cache,
                                   int64_t cache_row_stride_bytes, int64_t n_rows, int r, int d_rope,
                                   lkv_stream_t stream);

/*
 * Cache append into an FP8 cache: quantise the s_q new bf16 rows of every request (row b*s_q + i
 * of new_rows, laid out as for lkv_quantize_latent_fp8) into cache row cu_seqlens[b] + L_b - s_q + i
 * (the destinations of lkv_latent_cache_append).  A request with L_b < s_q or a destination past
 * cache_rows is skipped and recorded in the device error word.
 */
lkv_status lkv_latent_cache_append_fp8(const void* new_rows, int64_t new_row_stride, void* cache,
                                       int64_t cache_row_stride_bytes, int64_t cache_rows, int r,
                                       int d_rope, const int32_t* cu_seqlens, int batch, int s_q,
                                       lkv_stream_t stream);

/*
 * Merge attention results computed over disjoint key sets (split-KV combine):
 *   lse[r] = ln sum_p exp(lse_parts[p, r]);  out[r, :] = sum_p exp(lse_parts[p, r] - lse[r]) * o_parts[p, r, :]
 *   o_parts [n_parts, rows, d_v] fp32, lse_parts [n_parts, rows] fp32 (a part with lse = -inf
 *   holds no keys and is ignored); out [rows, d_v] in out_dtype; lse [rows] fp32 (may be NULL).
 * d_v must be a multiple of 4 and at most 1024.
 */
lkv_status lkv_merge_partials(const float* o_parts, const float* lse_parts, int n_parts,
                              int64_t rows, int d_v, int out_dtype, void* out, float* lse,
                              lkv_stream_t stream);

/*
 * Synchronise the current device and read the device error word (0 = none).  Returns
 * LKV_ERR_DEVICE if it is set, LKV_ERR_CUDA if synchronisation itself failed, else LKV_OK.
 * clear != 0 resets the word to 0 afterwards.  code_out may be NULL.
 */
lkv_status lkv_check_device(int32_t* code_out, int clear);

/*
 * The same check ordered on one stream only: waits for the work queued on `stream` so far
 * (cudaStreamSynchronize, not a device-wide synchronise, so other streams keep running), then
 * reads the device error word with a copy on that stream.  The word is shared by every stream of
 * the device, so it also shows failures recorded by other streams' finished kernels.
 * clear != 0 resets it to 0 on that stream afterwards.  code_out may be NULL.
 */
lkv_status lkv_check_stream(lkv_stream_t stream, int32_t* code_out, int clear);

/*
 * Failure-detection self test: launches one CTA that waits on an mbarrier no thread
 * arrives at, with the given limit.  The wait gives up, records LKV_SITE_SELFTEST in the
 * device error word and the kernel returns; the context stays usable.
 */
lkv_status lkv_selftest_wait_timeout(uint64_t limit_ns, lkv_stream_t stream);

/*
 * Projections either side of the decode path (GQLA explainer, section 2 "Methodology": the
 * absorbed path folds W_UK into the query and applies W_UV after attention; the GQA path expands
 * the latent into per-group keys and values).  j(h) = h / (h_q / groups).  bf16 operands, fp32
 * accumulation, bf16 results (dtype must be LKV_BF16, else LKV_ERR_UNSUPPORTED); all arrays are
 * contiguous device arrays unless a row stride is given.  Each call is one launch of the library's
 * tensor-core GEMM (tcgen05, TMA-fed, persistent over 128-row tiles); nothing is allocated.
 * Asynchronous on `stream`; a bounded wait that gives up is recorded in the device error word.
 *
 * lkv_absorb_query:    q [n_tok, h_q, d_h], w_uk [groups, r, d_h] -> q_abs [n_tok, h_q, r],
 *                      q_abs[t, h, :] = w_uk[j(h)] q[t, h, :]
 * lkv_unabsorb_output: o_lat [n_tok, h_q, r], w_uv [groups, r, d_v] -> out [n_tok, h_q, d_v],
 *                      out[t, h, :] = w_uv[j(h)]^T o_lat[t, h, :]
 * lkv_expand_latent:   c [n_rows, r] (row stride c_row_stride elements >= r), w [groups, r, d]
 *                      -> x [n_rows, groups, d],  x[t, j, :] = c[t, :] w[j]
 * Errors (checked before any launch): LKV_ERR_INVALID_ARG for NULL pointers, non-positive sizes,
 * h_q % groups != 0, leading dimensions beyond int range, operand pointers not 16-byte aligned, or
 * an operand row whose length or stride (d_h for absorb; r and d_v for unabsorb; c_row_stride and
 * d for expand) is not a multiple of 8 elements; LKV_ERR_CUDA if the launch fails.
 */
lkv_status lkv_absorb_query(const void* q, const void* w_uk, void* q_abs, int n_tok, int h_q, int groups,
                            int d_h, int r, int dtype, lkv_stream_t stream);
lkv_status lkv_unabsorb_output(const void* o_lat, const void* w_uv, void* out, int n_tok, int h_q,
                               int groups, int r, int d_v, int dtype, lkv_stream_t stream);
lkv_status lkv_expand_latent(const void* c, int64_t c_row_stride, const void* w, void* x, int64_t n_rows,
                             int groups, int r, int d, int dtype, lkv_stream_t stream);

/* Site codes stored in the device error word. */
#define LKV_SITE_SELFTEST 1
#define LKV_SITE_BAD_LENGTH 2     /* a request with L_b < s_q (append or decode)      */
#define LKV_SITE_BAD_ROW 3        /* a cache row past cache_rows                      */
#define LKV_SITE_WAIT_BASE 100    /* + kernel-specific wait site: a bounded wait gave up */

#ifdef __cplusplus
}
#endif

#endif /* LKV_H */
