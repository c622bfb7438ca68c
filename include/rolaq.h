/*
 * rolaq.h — C ABI of librolaq.so: a 2-bit rotated MLA latent cache on B200 (sm_100a).
 *
 * Method: "RoLaQ: Joint Rotation and Range Calibration for 2-Bit KV Caches in
 * Multi-Head Latent Attention" (arXiv 2610.20686v1).  Passages cited below by
 * page title and section:
 *   [S2.1]  §2.1 "One Cache, Two Roles": one content latent feeds K and V; the 64-d
 *           RoPE key k_R stays in BF16.
 *   [S3.2]  §3.2 "Response-Preserving Range Calibration": a per-layer threshold tau
 *           assigns standardized coordinates to four levels; the gain g scales the
 *           reconstruction around the group mean.
 *   [S3.3]  §3.3 "Joint Calibration and Inference": serving stores rotated latents as
 *           2-bit codes and folds the read-side rotation into the absorbed projections.
 *   [B.3]   §B.3: at the official threshold the MSE-optimal response is about 0.88;
 *           the coupled gain restores unit response.
 *   [S4.1]  §4.1 "Setup": protection keeps the first 4 sink and the most recent tokens
 *           in BF16.
 *   [S5.4]  §5.4 "Token Protection": sink plus recent-token budgets kept in BF16.
 *   [A.3]   §A.3 "Calibration and Storage": 288 B per unprotected token per layer
 *           (packed codes + group statistics + BF16 RoPE key); protected tokens also
 *           store BF16 content.
 *   [NB]    "2610.20686-rolaq-cache-accounting" notebook: 128 B of 2-bit codes +
 *           32 B of FP32 group statistics (two per 128-coordinate group) + 128 B BF16
 *           RoPE key = 288 B, versus 1152 B for BF16 MLA (4.000x ceiling).
 *
 * Conventions for every entry point:
 *   - All pointers named *_dev are device pointers owned by the caller; the library
 *     never allocates, frees or keeps them.  Host pointers are read during the call only.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  Work is
 *     enqueued asynchronously; the call returns once the kernels are launched.  The
 *     decode, write-path and projection kernels are launched as programmatic dependents
 *     of the previous work in the stream and wait for its completion before they read or
 *     write memory, so stream order holds as for ordinary launches; only their start-up
 *     overlaps the previous kernel's end.
 *   - Return value: ROLAQ_OK (0) or a negative ROLAQ_E* code.  Argument errors are
 *     detected on the host before anything is launched.  Errors that only the device can
 *     see (a page-table entry outside the pool) set bits in a device status word, skip
 *     the offending access and never trap; read them with rolaq_get_status().
 *   - bf16 means IEEE bfloat16 stored as uint16_t.
 */
#ifndef ROLAQ_H_
#define ROLAQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- fixed shapes [S2.1], [A.3], [NB] ------------------------------------------- */
#define ROLAQ_D_C          512   /* content-latent width                              */
#define ROLAQ_D_R          64    /* RoPE-key width                                    */
#define ROLAQ_D_NOPE       128   /* per-head no-RoPE query width (W_UK columns)       */
#define ROLAQ_D_V          128   /* per-head value width (W_UV columns)               */
#define ROLAQ_GROUP        128   /* coordinates per quantization group                */
#define ROLAQ_GROUPS       4     /* groups per token = D_C / GROUP                    */
#define ROLAQ_CODE_BYTES   128   /* 512 coordinates x 2 bit                           */
#define ROLAQ_META_BYTES   32    /* 4 groups x (mean, scale) fp32                     */
#define ROLAQ_KR_BYTES     128   /* 64 x bf16                                         */
#define ROLAQ_TOKEN_BYTES  288   /* CODE + META + KR                                  */
#define ROLAQ_BF16_TOKEN_BYTES 1152 /* (512 + 64) x bf16, the uncompressed MLA record */

/* ---- page layout ---------------------------------------------------------------
 * The cache is a pool of fixed-size pages.  A page holds ROLAQ_PAGE_TOKENS tokens of
 * one request as three planes (structure of arrays inside the page):
 *
 *   offset     0: codes [64 tokens][128 B]   byte b of a token holds coordinates
 *                                            4b..4b+3; coordinate j sits in bits
 *                                            2*(j%4)..2*(j%4)+1.  Code values 0..3 mean
 *                                            z < -tau, -tau <= z < 0, 0 <= z < tau,
 *                                            z >= tau (ascending level order).
 *   offset  8192: meta  [64 tokens][4 groups][2] fp32: (group mean, gain * group std)
 *   offset 10240: k_R   [64 tokens][64] bf16
 *
 * ROLAQ_PAGE_BYTES = 64 * 288 = 18432 = 144 rows of 128 B.  Token at logical position p
 * of request r lives in page page_table[r * max_pages_per_seq + p / 64] at row p % 64.
 * The pool base must be 1024-byte aligned (the decode kernel stages whole pages with
 * a 128-byte-swizzled tensor copy).
 * ------------------------------------------------------------------------------- */
#define ROLAQ_PAGE_TOKENS  64
#define ROLAQ_PAGE_BYTES   18432
#define ROLAQ_PAGE_CODES_OFFSET 0
#define ROLAQ_PAGE_META_OFFSET  8192
#define ROLAQ_PAGE_KR_OFFSET    10240

/* Rotation operand prepared by rolaq_prepare_rotation: three bf16 planes [3][512][512]. */
#define ROLAQ_RSPLIT_BYTES (3u * 512u * 512u * 2u)

/* ---- error codes ---------------------------------------------------------------- */
#define ROLAQ_OK            0
#define ROLAQ_EINVAL       -1   /* null / misaligned pointer, bad size or shape        */
#define ROLAQ_ENOSPACE     -2   /* workspace smaller than rolaq_decode_workspace_bytes */
#define ROLAQ_ECUDA        -3   /* a CUDA runtime or driver call failed                */
#define ROLAQ_EUNSUPPORTED -4   /* shape the kernels do not implement (heads % 16)     */

/* Device status bits reported by rolaq_get_status(). */
#define ROLAQ_STATUS_BAD_PAGE   1  /* page-table entry < 0 or >= num_pages (skipped)  */
#define ROLAQ_STATUS_BAD_SLOT   2  /* append target outside its request's pages, or (BF16
                                      decode) a position without a bf16 copy          */
#define ROLAQ_STATUS_TIMEOUT    4  /* a pipeline wait gave up (results of that call invalid) */
#define ROLAQ_STATUS_RANGE      8  /* a decoded x or a query element beyond the fp16 range
                                      (|x|, |q| >= 65504): that decode result is invalid  */

/* Cache descriptor.  Plain data; the caller owns every buffer it points to.
 *   pages_dev       page pool, num_pages * ROLAQ_PAGE_BYTES bytes, 1024-B aligned.
 *   page_table_dev  int32 [batch][max_pages_per_seq]; entry = page index in the pool.
 *   prot_dev        optional BF16 side store [batch][n_sink + n_recent][512] holding the
 *                   rotated content of protected tokens [S4.1], [A.3]; NULL when
 *                   n_sink + n_recent == 0.  Row p (p < n_sink) holds sink position p;
 *                   row n_sink + (p % n_recent) holds recent position p.               */
typedef struct rolaq_cache {
    void*          pages_dev;
    int64_t        num_pages;
    const int32_t* page_table_dev;
    int32_t        batch;
    int32_t        max_pages_per_seq;
    void*          prot_dev;
    int32_t        n_sink;
    int32_t        n_recent;
} rolaq_cache;

/* Per-layer quantizer constants, fixed during serving [S3.3].
 *   level_a, level_b: the four reconstruction levels are -b, -a, +a, +b, the centroids
 *   of a standard normal on [0, tau) and [tau, inf) mirrored [S3.2].                 */
typedef struct rolaq_layer_params {
    float tau;
    float gain;
    float level_a;
    float level_b;
} rolaq_layer_params;

/* Fill p for threshold tau > 0 and gain > 0.  The levels are computed on the host in
 * double (a = (phi(0) - phi(tau)) / (Phi(tau) - 1/2), b = phi(tau) / (1 - Phi(tau)))
 * and rounded to fp32 once.  Returns ROLAQ_EINVAL for a non-finite or non-positive
 * tau or gain.  [S3.2]                                                                */
int rolaq_layer_params_init(rolaq_layer_params* p, float tau, float gain);

/* Coupled gain for threshold tau > 0 [S3.2], [B.3]: the gain links to the threshold so
 * that the centered reconstruction has unit response.  With z ~ N(0, 1) and the centroid
 * levels of tau, the response of the reconstruction gain * level(z) is
 *   kappa(tau) = gain * E[z * level(z)] = gain * 2 (a (phi(0) - phi(tau)) + b phi(tau)),
 * so the coupled gain is 1 / E[z * level(z)].  Computed on the host in double.  Writes the
 * coupled gain to *gain and, when kappa1 is not NULL, E[z * level(z)] (the response at
 * gain 1; about 0.8825 at the Lloyd-Max threshold 0.9816, where the coupled gain is
 * about 1.1331) to *kappa1.  Returns ROLAQ_EINVAL for a NULL gain or a non-finite or
 * non-positive tau.  Pass the result to rolaq_layer_params_init as the layer's gain.      */
int rolaq_coupled_gain(float tau, double* gain, double* kappa1);

/* Convert the fp32 rotation R_dev [512][512] (row-major, y = c . R for a row vector c)
 * into the tensor-core operand R_split_dev (ROLAQ_RSPLIT_BYTES, 16-B aligned): plane 0
 * holds bf16(R^T), plane 1 the nearest bf16 of R^T - plane0, plane 2 the nearest bf16 of
 * what is left, each [512 out][512 in].  The three planes reproduce R to about 2^-26
 * relative, so y keeps fp32-level accuracy.  Run once per layer at load time.  [S3.3]                                                         */
int rolaq_prepare_rotation(const float* R_dev, void* R_split_dev, void* stream);

/* Write path [S3.2], [S3.3], [A.3]: for each of n tokens i, rotate c_dev[i] (bf16 [n][512])
 * by R, split into 4 groups of 128, standardise each group by its fp32 mean and
 * population std, assign 2-bit codes by tau, pack, and store (mean, gain*std) and the
 * bf16 RoPE key k_R_dev[i] ([n][64]) into the page of request req_dev[i] at logical
 * position pos_dev[i].  With protection configured, the token's bf16 rotated content is
 * also written to the side store when pos < n_sink (sink row) or
 * pos >= seq_lens_dev[req] - n_recent (recent ring row), where seq_lens_dev (int32
 * [batch], may be NULL when n_recent == 0) holds each request's length after this
 * append.  A group with zero spread gets code 2 and scale 0.  Targets outside the page
 * table set ROLAQ_STATUS_BAD_SLOT and are skipped.  n == 0 is a no-op.               */
int rolaq_quantize_append(const rolaq_cache* cache, const rolaq_layer_params* p,
                          const void* R_split_dev, const void* c_dev, const void* k_R_dev,
                          const int32_t* req_dev, const int32_t* pos_dev,
                          const int32_t* seq_lens_dev, int n, void* stream);

/* Bytes of device workspace rolaq_decode_attn needs for `batch` requests and `heads`
 * query heads on the current device (split-K partials and their merge state):
 * (SM count + batch) x heads x 2,056 bytes; 0 for batch <= 0 or heads not a positive
 * multiple of 16.                                                                      */
size_t rolaq_decode_workspace_bytes(int batch, int heads);

/* Read path [S2.1], [S3.3]: absorbed-MLA decode attention straight from the packed cache.
 * For request r with L = seq_lens_dev[r] tokens and head h:
 *   x_t      = mean_g + scale_g * level(code)      (2-bit token)  or the bf16 side-store
 *              row (protected token: t < n_sink, or t >= L - n_recent)
 *   s_t      = (q_c_rot[r,h] . x_t + q_R[r,h] . k_R_t) * sm_scale
 *   out[r,h] = sum_t softmax(s)_t x_t                (rotated basis; the inverse rotation
 *              belongs to the absorbed value projection [S3.3])
 *   lse[r,h] = log sum_t exp(s_t)                    (natural log)
 * q_c_rot_dev bf16 [batch][heads][512] already carries R (q . W_UK . R), q_R_dev bf16
 * [batch][heads][64]; out_dev fp32 [batch][heads][512]; lse_dev fp32 [batch][heads]
 * (may be NULL).  heads must be a positive multiple of 16, batch <= cache->batch.
 * L == 0 gives out = 0 and lse = -inf.  workspace_dev (16-B aligned) must hold
 * rolaq_decode_workspace_bytes(batch, heads) bytes; it is scratch owned by the caller
 * and needs no initialisation.  Split-K over the sequence with a log-sum-exp merge.
 * Arithmetic: x_t, q_c_rot and the probabilities enter the tensor-core products as fp16
 * (k_R and q_R as bf16); scores, sums and out accumulate in fp32.  A token whose
 * |mean| + scale * level_b, or a query element whose magnitude, reaches 65504 sets
 * ROLAQ_STATUS_RANGE.                                                                */
int rolaq_decode_attn(const rolaq_cache* cache, const rolaq_layer_params* p,
                      const void* q_c_rot_dev, const void* q_R_dev,
                      const int32_t* seq_lens_dev, int batch, int heads, float sm_scale,
                      float* out_dev, float* lse_dev,
                      void* workspace_dev, size_t workspace_bytes, void* stream);

/* BF16 decode on the same cache [S4.1], [A.3]: quantisation disabled, every token read
 * from its bf16 copy in the side store (the content the protected tokens keep) with its
 * RoPE key from the page; the 2-bit codes are not read.  Result as rolaq_decode_attn for
 * a cache whose every token is protected; arguments, workspace and errors as
 * rolaq_decode_attn, and in addition: the cache must have a side store (else
 * ROLAQ_EINVAL) with n_sink and n_recent multiples of 64 (else ROLAQ_EUNSUPPORTED), so
 * that each 64-token page maps to one run of side-store rows.  A request with
 * L > n_sink + n_recent has positions without a bf16 copy: ROLAQ_STATUS_BAD_SLOT is set
 * and its result is not valid.  Arithmetic: x, q_c_rot and the probabilities enter the
 * tensor-core products as bf16 (both operands of one product share a type), sums fp32.
 * Each page is moved with bulk tensor copies (64 side-store rows as eight 64 x 64 boxes
 * with the 128-byte swizzle, plus the page's 64 RoPE rows): 1,152 B per token.          */
int rolaq_decode_attn_bf16(const rolaq_cache* cache, const rolaq_layer_params* p,
                           const void* q_c_rot_dev, const void* q_R_dev,
                           const int32_t* seq_lens_dev, int batch, int heads, float sm_scale,
                           float* out_dev, float* lse_dev,
                           void* workspace_dev, size_t workspace_bytes, void* stream);

/* Bytes of device workspace rolaq_decode_attn_append needs: rolaq_decode_workspace_bytes
 * plus batch x 2,048 (the new tokens' rotated coordinates, fp32 [batch][512]); 0 where
 * rolaq_decode_workspace_bytes is 0.                                                   */
size_t rolaq_decode_append_workspace_bytes(int batch, int heads);

/* Serving step with the per-step write fused into the decode [S4.1], [S5.4],
 * [A.3]: one new token per request is appended (recent tokens stay protected in bf16,
 * older ones live as 2-bit codes) and the decode runs over the cache that includes it,
 * in the two launches of one decode call.  For request r with L = seq_lens_dev[r] >= 1
 * (the length AFTER the append) the token at position L - 1 is written as
 * rolaq_quantize_append with req = r, pos = L - 1 and these seq_lens writes it (codes,
 * statistics, k_R, and its side-store row when protected), from row r of c_new_dev
 * (bf16 [batch][512]) and k_R_new_dev (bf16 [batch][64]); R_split_dev is the operand of
 * rolaq_prepare_rotation.  out and lse are those of rolaq_decode_attn over the L tokens:
 * the new token enters with the value the decode reads from the cache (bf16 y when
 * protected, else the fp16 mean + scale * level) and a score summed in fp32.  A request
 * with L <= 0 gets nothing written, out = 0 and lse = -inf.  workspace_dev (16-B
 * aligned) must hold rolaq_decode_append_workspace_bytes(batch, heads) bytes and needs
 * no initialisation.  Errors as rolaq_decode_attn; a null or misaligned (16 B)
 * R_split_dev, c_new_dev or k_R_new_dev gives ROLAQ_EINVAL.  A position whose page is
 * not mapped in page_table sets ROLAQ_STATUS_BAD_SLOT and is not stored; the decode
 * still counts the token.  How the work is spread: in the split kernel one otherwise
 * idle warp of every CTA computes a few coordinates of y = c . R for all new tokens (so
 * R is read once, spread over the SMs); the merge kernel, which runs after it, finishes
 * the write and adds the new token's term.  Calls that overlap on the GPU must not share
 * a workspace or append to the same request.                                            */
int rolaq_decode_attn_append(const rolaq_cache* cache, const rolaq_layer_params* p,
                             const void* R_split_dev, const void* c_new_dev, const void* k_R_new_dev,
                             const void* q_c_rot_dev, const void* q_R_dev,
                             const int32_t* seq_lens_dev, int batch, int heads, float sm_scale,
                             float* out_dev, float* lse_dev,
                             void* workspace_dev, size_t workspace_bytes, void* stream);

/* Decode without a caller-provided workspace.  Same arguments, result and errors as
 * rolaq_decode_attn, except that the split-K scratch lives in a fixed array inside the
 * library (ROLAQ_STATIC_SCRATCH_BYTES per GPU, held by every GPU that loads the library
 * until the process exits) instead of caller memory.  It is for callers that cannot call
 * cudaMalloc: code running while a memory pool or a captured allocator owns the device
 * memory, plug-ins that are handed tensors but no allocator, and hosts that forbid
 * allocation after start-up.  The call itself allocates nothing.
 *   - The array is part of the library's device code, so the 32 MiB are committed on a
 *     device when the library's module is loaded there: at the first call of any librolaq
 *     entry point that reaches that device (with lazy module loading), not only at the
 *     first call of this one.  Every process that loads the library pays it on each device
 *     it uses, whether or not it calls this entry point.  ROLAQ_ECUDA from the first call
 *     on a device can mean that this load failed (for instance because a memory pool
 *     already holds nearly all of the device's memory).
 *   - The first call on each device looks up the array's device address on that device;
 *     make that first call before any stream capture.
 *   - The split-K plan uses as many work items as the array holds, up to one per SM:
 *     (items + batch) x heads x 2,056 bytes <= ROLAQ_STATIC_SCRATCH_BYTES.  A call for
 *     which not even one item fits ((1 + batch) x heads x 2,056 bytes above it) returns
 *     ROLAQ_ENOSPACE before anything is launched.
 *   - Every call on a device shares the one array and leaves its contents behind; the
 *     kernels overwrite whatever they read, so nothing needs clearing, but calls that can
 *     overlap on the GPU (different streams without ordering between them) race on it.
 * The paper has no counterpart of this entry point; it is an integration convenience.   */
#define ROLAQ_STATIC_SCRATCH_BYTES (32u * 1024u * 1024u)
int rolaq_decode_attn_static(const rolaq_cache* cache, const rolaq_layer_params* p,
                             const void* q_c_rot_dev, const void* q_R_dev,
                             const int32_t* seq_lens_dev, int batch, int heads, float sm_scale,
                             float* out_dev, float* lse_dev, void* stream);

/* ---- absorbed projections around the cache [S3.3], [Fig. 3a] ---------------------
 * The read-side rotation never runs per token: R folds into the absorbed query
 * projection and R^T into the absorbed value projection, so the decode works in the
 * rotated basis and the caller's projections see the original one.  The folded weights
 * are bf16 (computed in fp32, rounded once).  All pointers are device memory owned by the
 * caller, dense and row-major as listed; alignment: the folded weights and the per-step
 * inputs 16 bytes, fp32 arrays otherwise 4 and bf16 outputs 2.  NULL or misaligned
 * pointers, heads <= 0 (or above 65535) and batch < 0 give ROLAQ_EINVAL and launch
 * nothing.  batch == 0 makes the per-step calls a no-op that returns ROLAQ_OK without
 * looking at the pointers (empty tensors may carry NULL).                              */

/* Once per layer: W_q[h] = W_UK[h]^T . R and W_o[h] = R^T . W_UV[h] (fp32 sums).
 * W_UK_dev, W_UV_dev fp32 [heads][512][128] (latent row k, head column n: the up
 * projections c . W_UK[h] -> k_nope, c . W_UV[h] -> v); R_dev fp32 [512][512] with
 * y = c . R; W_q_dev bf16 [heads][128][512]; W_o_dev bf16 [heads][512][128].         */
int rolaq_fold_weights(const float* W_UK_dev, const float* W_UV_dev, const float* R_dev,
                       int heads, void* W_q_dev, void* W_o_dev, void* stream);

/* Per decode step: q_c_rot[b][h] = q_nope[b][h] . W_q[h], the query rolaq_decode_attn
 * takes.  q_nope_dev bf16 [batch][heads][128]; W_q_dev bf16 from rolaq_fold_weights;
 * q_c_rot_dev bf16 [batch][heads][512].  Tensor-core product of the bf16 operands with
 * fp32 accumulation, rounded to bf16 (nearest even) once.                            */
int rolaq_fold_query(const void* q_nope_dev, const void* W_q_dev, int batch, int heads,
                     void* q_c_rot_dev, void* stream);

/* Per decode step: v[b][h] = out[b][h] . W_o[h], the attention output back in the
 * original basis and through the value up-projection.  out_dev fp32 [batch][heads][512]
 * (rolaq_decode_attn's output); W_o_dev bf16 from rolaq_fold_weights; v_dev fp32
 * [batch][heads][128].  out enters the tensor-core product rounded to bf16 (nearest
 * even); the sums accumulate in fp32.                                                 */
int rolaq_unfold_output(const float* out_dev, const void* W_o_dev, int batch, int heads,
                        float* v_dev, void* stream);

/* Copy the device status word of the current device to *bits and clear it.  Blocks until
 * `stream` has finished.                                                              */
int rolaq_get_status(int* bits, void* stream);

/* Static description of an error code. */
const char* rolaq_strerror(int code);

/* Library version, major * 10000 + minor * 100 + patch. */
int rolaq_version(void);

#ifdef __cplusplus
}
#endif
#endif /* ROLAQ_H_ */
