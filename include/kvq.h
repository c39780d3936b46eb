/*
 * kvq.h -- C ABI of the B200 (sm_100a) rotated-token KV-cache quantizer.
 *
 * The method (TurboQuant form, calibration free):
 *   quantize  x -> ||x||, z = H (delta .* x) / ||x||, b-bit Lloyd-Max codes
 *             of z (for N(0,1), or for the exact Beta law of a rotated unit
 *             coordinate with KVQ_BETA_CODEBOOK), residual r = z - c[code],
 *             1-bit QJL sketch sign(S r), fp16 norms (||x||, ||r||);
 *             optionally behind the NSN front end (kvq_nsn_quantize);
 *   decode    rotate each query once, logits straight from the packed codes
 *             plus the QJL correction, softmax, weighted sum of the decoded
 *             values, all over the packed cache (plain or NSN), optionally
 *             followed by an fp16 residual window of the newest tokens.
 * Sources: "O Que E TurboQuant?" (TurboQuant blog), sections "Estagio 1:
 * Rotacao Aleatoria + Compressao PolarQuant", "Estagio 2: Correcao Residual
 * QJL" and "Como Implementar"; "PolarQuant: Optimal Gaussian Weight
 * Quantization via Hadamard Rotation for LLM Compression", section 2
 * (block normalisation, Walsh-Hadamard rotation, Gaussian Lloyd-Max,
 * dequantisation); "NSNQuant: A Double Normalization Approach for
 * Calibration-Free Low-Bit Vector Quantization of KV Cache", sections 1, 2
 * and 4 (Normalize-Shift-Normalize front end, RHT, block flush).
 *
 * Conventions for every entry point:
 *  - Return 0 (KVQ_OK) on success or a negative KVQ_E* code; the message of
 *    the last failure on the calling thread is kvq_last_error().  Nothing is
 *    thrown across the ABI and no kernel traps.
 *  - A handle belongs to the CUDA device that was current at kvq_init.
 *    Every call that launches work or reads the device (all but kvq_init,
 *    kvq_destroy, kvq_codebook, kvq_get_info, kvq_get_constants and
 *    kvq_last_error) requires that device to be current and returns
 *    KVQ_EINVAL, before any launch, when another device is current.
 *  - Pointer arguments named as "device" must point to device memory of the
 *    current CUDA device; the caller allocates and owns every input, output
 *    and workspace buffer.  The handle owns only its constants.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls other than kvq_init / kvq_destroy / kvq_status /
 *    kvq_get_constants are asynchronous on that stream and do not
 *    synchronise.
 *  - Errors in arguments are detected on the host before any launch
 *    (KVQ_EINVAL / KVQ_EUNSUPPORTED) and leave outputs untouched.
 *    Conditions found on the device (non-finite input, an fp16 norm
 *    overflow, a bounded wait that gave up) are ORed into the handle's
 *    device status word and reported by kvq_status().
 *
 * Packed cache layout.  A "stream" is a sequence of vectors of one head
 * (one call of kvq_quantize, or one (batch, kv-head) of a cache).  For
 * vector t of a stream, with L = 2^b levels, m = d projection rows:
 *   codes  uint32 [t][b][d/32]  bit i of word (p, w) = bit p of the code of
 *                               coordinate 32*w + i (bit planes);
 *   qjl    uint32 [t][m/32]     bit i of word w = [ (S r)_{32w+i} >= 0 ];
 *   norms  fp16   [t][2]        (||x||, ||r||)  -- NSN: (||x||, ||w||).
 * Coordinates are in the rotated domain, Sylvester (natural) order.
 *
 * KVQ_LAYOUT_BLOCK32 stores the same bits transposed per block of 32
 * consecutive vectors (vector t is bit t % 32 of block t / 32), the layout
 * the decode kernel consumes for values (its value sums contract over
 * tokens, four tokens per tensor-core register):
 *   codes  uint32 [blk][b][d]   bit i of word (blk, p, j) = bit p of the code
 *                               of coordinate j of vector 32*blk + i;
 *   qjl    uint32 [blk][m]      bit i of word (blk, k) = QJL bit of row k of
 *                               vector 32*blk + i;
 *   norms  fp16   [t][2]        as above (one record per vector).
 * Bits of vectors past the end of the input are 0.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---------------------------------------------------- */
#define KVQ_OK 0
#define KVQ_EINVAL (-1)       /* bad argument: null/misaligned pointer, size, dtype, layout */
#define KVQ_EUNSUPPORTED (-2) /* valid by the method but not built (e.g. fp32 input at d = 256) */
#define KVQ_ECUDA (-3)        /* a CUDA runtime/driver call failed (message has the CUDA error) */
#define KVQ_ENOMEM (-4)       /* device or host allocation failed in kvq_init */
#define KVQ_ENONFINITE (-5)   /* kvq_status: an input was NaN/Inf or a norm overflowed fp16 */
#define KVQ_ETIMEOUT (-6)     /* kvq_status: a kernel's bounded wait gave up; outputs invalid */

/* ---- flags of kvq_init ------------------------------------------------- */
#define KVQ_QJL 1u            /* store the 1-bit QJL residual sketch (m = d rows) */
/* Codebook: Lloyd-Max for the exact law of one coordinate of a rotated unit
 * vector scaled by sqrt(d) (Beta((d-1)/2, (d-1)/2) on [-1, 1], stretched to
 * [-sqrt(d), sqrt(d)]; TurboQuant blog, "Estágio 1") instead of N(0, 1). */
#define KVQ_BETA_CODEBOOK 2u
/* Rotation on the CUDA cores: kvq_quantize / kvq_quantize_batch with 16-bit
 * input, wherever the tensor-core product X (H D)^T would run (d <= 128, and
 * d = 256 without KVQ_QJL), rotate by the in-register Walsh-Hadamard
 * transform instead (the kernel that fp32 input and d = 256 with QJL use).
 * Same outputs under the same rules (codes exact outside the decision-level
 * band, norms within one fp16 ulp); one launch per job.  For comparing the
 * two rotations at one configuration; the NSN entry points ignore it. */
#define KVQ_CUDA_CORE_ROTATION 4u

/* ---- element types of inputs ------------------------------------------ */
#define KVQ_F32 0
#define KVQ_F16 1
#define KVQ_BF16 2

/* ---- packed layouts ------------------------------------------------------ */
#define KVQ_LAYOUT_TOKEN 0    /* one record per vector (see "Packed cache layout") */
#define KVQ_LAYOUT_BLOCK32 1  /* bit planes transposed in blocks of 32 consecutive vectors */

/* Device status word bits, as returned in *bits by kvq_status. */
#define KVQ_STATUS_NONFINITE 1u
#define KVQ_STATUS_NORM_OVERFLOW 2u
#define KVQ_STATUS_TIMEOUT 4u

typedef struct kvq_ctx* kvq_handle;

/*
 * kvq_init -- build the constants of one quantizer and upload them to the
 * current device (TurboQuant blog, "Como Implementar": codebooks are
 * precomputed per head dimension and bit width; no calibration data).
 *   h      out: new handle (host pointer to a kvq_handle).
 *   d      head dimension, one of 64, 128, 256 (power of two: FWHT).
 *   b      Lloyd-Max bits per coordinate, 1..4.
 *   seed   seeds the SplitMix64 streams: Rademacher signs use `seed`, the
 *          Gaussian projection S (d x d, rounded to fp16) uses `seed + 1`.
 *   flags  KVQ_QJL, KVQ_BETA_CODEBOOK and/or KVQ_CUDA_CORE_ROTATION, or 0.
 * Synchronous.  Allocates device memory for the constants and a status
 * word.  Errors: KVQ_EINVAL, KVQ_ENOMEM, KVQ_ECUDA.
 */
int kvq_init(kvq_handle* h, int d, int b, uint64_t seed, uint32_t flags);

/*
 * kvq_codebook -- the codebook a handle with (d, b, flags) uses, computed on
 * the host (no device needed): 2^b ascending centroids and the 2^b - 1
 * decision levels between them (the midpoints), rounded to fp32.
 *   centroids   host, 2^b floats;  thresholds  host, 2^b - 1 floats.
 * Errors: KVQ_EINVAL (d, b, flags as kvq_init; null outputs).
 */
int kvq_codebook(int d, int b, uint32_t flags, float* centroids, float* thresholds);

/* kvq_destroy -- free the handle and its device constants (synchronous).
 * A NULL handle is accepted and ignored. */
int kvq_destroy(kvq_handle h);

/*
 * kvq_quantize -- quantize n vectors (TurboQuant blog, Stages 1 and 2;
 * PolarQuant section 2).  Per vector x (row i of x):
 *   norm = ||x||; z = H (delta .* x) / norm; code_j = #{k : z_j >= t_k};
 *   r = z - c[code]; gamma = ||r||; qjl bit_i = [(S r)_i >= 0];
 *   norms = (fp16(norm), fp16(gamma)).  A zero vector stores all zeros.
 *   x      device, n rows of d elements of `dtype`, row stride `ld`
 *          elements (ld >= d; ld * element size a multiple of 16 bytes;
 *          x 16-byte aligned).
 *   n      number of vectors, >= 0 (0 is a no-op).
 *   layout KVQ_LAYOUT_TOKEN or KVQ_LAYOUT_BLOCK32 (codes and qjl).
 *   codes  device, 16-byte aligned; n * b * d/32 uint32 (token layout) or
 *          ceil(n/32) * b * d uint32 (block-32 layout).
 *   qjl    device, 16-byte aligned, n * d/32 (token) or ceil(n/32) * d
 *          (block-32) uint32; must be NULL when the handle has no KVQ_QJL
 *          flag and non-NULL when it has.
 *   norms  device, n * 2 fp16 (bit patterns), 4-byte aligned.
 * fp32 input is built for d <= 128.  Non-finite inputs and norms above the
 * fp16 range set status bits; those rows' outputs are unspecified.
 */
int kvq_quantize(kvq_handle h, const void* x, int dtype, int64_t n, int64_t ld, int layout, uint32_t* codes,
                 uint32_t* qjl, uint16_t* norms, void* stream);

/* One stream of vectors for kvq_quantize_batch: the arguments of
 * kvq_quantize, with the same meaning and rules. */
typedef struct kvq_quant_job {
    const void* x;
    int dtype;
    int64_t n;
    int64_t ld;
    int layout;
    uint32_t* codes;
    uint32_t* qjl;
    uint16_t* norms;
} kvq_quant_job;

/*
 * kvq_quantize_batch -- kvq_quantize of `count` streams of vectors (for
 * instance the keys and the values of one layer) in as few launches as the
 * kernels allow: two consecutive non-empty jobs of the same 16-bit dtype
 * share one launch (at d <= 128, and at d = 256 without KVQ_QJL), whose
 * tiles are those of the first job then those of the second; the others
 * take one launch each.  The outputs are exactly those of one kvq_quantize
 * call per job.
 *   count  >= 0; jobs  host array of `count` descriptors (read during the
 *          call only).  Every job is checked before anything is launched;
 *          an error names the job ("job i: ...") and launches nothing.
 * Asynchronous on `stream`.  Errors: as kvq_quantize.
 */
int kvq_quantize_batch(kvq_handle h, int count, const kvq_quant_job* jobs, void* stream);

/*
 * kvq_nsn_quantize -- NSN front end then the quantizer without QJL
 * (NSNQuant section 1 Normalize-Shift-Normalize, section 2 Hadamard, section
 * 4 block flush).  For each head and each block of 128 consecutive tokens:
 *   u_t = sqrt(d) x_t / ||x_t|| (0 for a zero token); o = mean_t u_t per
 *   channel, stored as fp16; w_t = u_t - fp16(o); w_t is quantized as above
 *   (codes of H (delta .* w_t) / ||w_t||); norms = (fp16 ||x_t||,
 *   fp16 ||w_t||), i.e. s1 = ||x||/sqrt(d), s2 = ||w||/sqrt(d).
 *   x           device, [n_heads][n_tok][d] contiguous, dtype as above.
 *   n_tok       tokens per head, a multiple of 128 (the full-precision tail
 *               of a real cache stays outside, NSNQuant section 4).
 *   layout      KVQ_LAYOUT_TOKEN (keys) or KVQ_LAYOUT_BLOCK32 (values; blocks
 *               of 32 tokens never straddle heads since n_tok % 128 == 0).
 *   codes       device, n_heads * n_tok * b * d/32 uint32.
 *   norms       device, n_heads * n_tok * 2 fp16.
 *   block_mean  device, n_heads * (n_tok/128) * d fp16.
 * Requires a handle without KVQ_QJL (KVQ_EINVAL otherwise); at d = 256 the
 * input must be fp16 or bf16 (fp32 returns KVQ_EUNSUPPORTED).
 */
int kvq_nsn_quantize(kvq_handle h, const void* x, int dtype, int64_t n_heads, int64_t n_tok, int layout,
                     uint32_t* codes, uint16_t* norms, uint16_t* block_mean, void* stream);

/* One packed cache (keys or values) of batch * hkv streams, each holding up
 * to `capacity` vectors in the layout above; stream (bi, hi) starts at
 * vector (bi * hkv + hi) * capacity.  Keys use KVQ_LAYOUT_TOKEN, values
 * KVQ_LAYOUT_BLOCK32; capacities are multiples of 32 and the buffers 16-byte
 * aligned. */
typedef struct kvq_cache {
    const uint32_t* codes;  /* device, streams * capacity * b * d/32 */
    const uint32_t* qjl;    /* device, streams * capacity * d/32; NULL without KVQ_QJL */
    const uint16_t* norms;  /* device, streams * capacity * 2 fp16 */
    int64_t capacity;       /* vectors per stream, >= max_T */
    int32_t layout;         /* KVQ_LAYOUT_TOKEN (keys) or KVQ_LAYOUT_BLOCK32 (values) */
} kvq_cache;

/* Bytes of device workspace a decode call (kvq_decode_attend,
 * kvq_nsn_decode_attend, kvq_decode_attend_ex with or without a residual
 * window) needs for these sizes; computed on the host, no device work. */
size_t kvq_decode_workspace(kvq_handle h, int batch, int hq, int hkv, int64_t max_T);

/*
 * kvq_decode_attend -- one decode step of attention over packed K and V
 * caches (TurboQuant blog, "Como Implementar": queries rotated once,
 * logits computed straight from the indices; PolarQuant section 2
 * dequantisation moved to the query side).  For query head g of batch bi,
 * attending KV head hi = g / (hq / hkv) over tokens t < seq_len[bi]:
 *   q' = H (delta .* q); p = S q'  (fp32)
 *   l_t = scale * (n_t / d) * ( sum_j q'_j c[code_tj]
 *                               + sqrt(pi/2)/m * gamma_t * sum_i p_i (2 bit_ti - 1) )
 *   softmax over t (split over the context, merged exactly);
 *   out = 1/(d sum_t w_t) * delta .* H ( sum_t w_t n_t c[vcode_t]
 *           + sqrt(pi/2)/m * S^T sum_t w_t n_t gamma_t (2 vbit_t - 1) ).
 *   q        device, [batch][hq][d] of `dtype`, contiguous.
 *   hq, hkv  query and KV heads; hq a multiple of hkv, hq/hkv in {1,2,4,8}.
 *   k, v     host pointers to cache descriptors (device buffers inside).
 *   seq_len  device, int32 [batch], each in [0, max_T]; 0 gives a zero output.
 *   max_T    bound on seq_len (sizes the split grid), <= capacity.
 *   scale    logit scale (e.g. 1/sqrt(d)).
 *   logits   device, fp32 [batch][hq][max_T] or NULL; entries past seq_len
 *            are written as -inf.
 *   out      device, fp32 [batch][hq][d].
 *   workspace, ws_bytes  device scratch of at least
 *            kvq_decode_workspace(h, batch, hq, hkv, max_T) bytes, 16-byte
 *            aligned; contents on entry are ignored.
 */
int kvq_decode_attend(kvq_handle h, const void* q, int dtype, int batch, int hq, int hkv,
                      const kvq_cache* k, const kvq_cache* v, const int32_t* seq_len, int64_t max_T,
                      float scale, float* logits, float* out, void* workspace, size_t ws_bytes,
                      void* stream);

/* Bytes of the fixed decode scratch built into the library (see
 * kvq_decode_attend_noalloc). */
#define KVQ_NOALLOC_SCRATCH_BYTES (8u << 20)

/*
 * kvq_nsn_decode_attend -- kvq_decode_attend over caches written by
 * kvq_nsn_quantize (NSNQuant section 4: attention straight from the stored
 * byproducts).  A stored vector stands for
 *   x_hat = ||x||/sqrt(d) (w_hat + o_blk),
 * where w_hat is the codebook vector rotated back and scaled to ||w|| (the
 * plain dequantization with norm ||w||), and o_blk is the fp16 mean of its
 * block of 128 tokens.  So
 *   l_t = scale ||x_t||/sqrt(d) (||w_t||/d <q', c[code_t]> + <q, o_blk(t)>),
 *   out = sum_t p_t x_hat(v_t).
 * Arguments as kvq_decode_attend, and:
 *   k, v          norms hold (fp16 ||x||, fp16 ||w||); codes as usual; no QJL.
 *   k_block_mean, v_block_mean
 *                 device, fp16; per stream capacity/128 blocks of d, stream
 *                 (bi, hi) at block (bi * hkv + hi) * capacity/128, 16-byte
 *                 aligned.  Capacities must be multiples of 128.
 * The workspace size is kvq_decode_workspace's.  Requires a handle without
 * KVQ_QJL (KVQ_EINVAL); every (d, b) is built (b <= 2, and b = 3 at d <= 128,
 * on the tensor-core path, the rest on the CUDA cores).
 */
int kvq_nsn_decode_attend(kvq_handle h, const void* q, int dtype, int batch, int hq, int hkv, const kvq_cache* k,
                          const kvq_cache* v, const uint16_t* k_block_mean, const uint16_t* v_block_mean,
                          const int32_t* seq_len, int64_t max_T, float scale, float* logits, float* out,
                          void* workspace, size_t ws_bytes, void* stream);

/*
 * Double-quantized NSN side data (NSNQuant section 3, "Double Quantization":
 * the NSN parameters -- the mean o and the scale s1 -- are themselves stored
 * with 4 bits).  The pages give no format; this library's, per block of 128
 * tokens of one head, is one side record of kvq_nsn_dq_side_bytes(d) bytes:
 *   bytes [0,2) fp16 lo, [2,4) fp16 step, [4,6) fp16 nstep, [6,8) zero;
 *   [8, 8 + d/2)        4-bit codes q_j of the block means (byte i: channel
 *                       2i in the low nibble, 2i+1 in the high one);
 *   [8 + d/2, + 64)     4-bit codes q_t of the 128 token norms (byte i: token
 *                       2i low nibble, 2i+1 high);
 *   zero padding to a multiple of 16 bytes (144 bytes at d = 128, 112 at 64,
 *   208 at 256).
 * The stored values are   n1_t = q_t nstep   (q_t = 0 only for a zero token)
 *                         o_hat_j = fp32(lo + step q_j)   (one rounding),
 * and the transform uses them: u_t = sqrt(d) x_t / n1_t, w_t = u_t - o_hat,
 * so a token is exactly n1_t/sqrt(d) (w_t + o_hat) before w_t is coded.
 * Codes:  nstep = fp16(max_t ||x_t|| / 15), q_t = clamp(rint(||x_t||/nstep),
 * 1, 15);  lo = fp16(min_j o_j), step = fp16((max_j o_j - min_j o_j) / 15),
 * q_j = clamp(rint((o_j - lo) / step), 0, 15) (0 when step = 0);  o is the
 * block mean of u.  Per token only fp16 ||w_t|| is stored besides the codes:
 * 0.195 bits per element of side data at d = 128 with 128-token blocks,
 * against 0.375 with fp16 ||x||, ||w|| and fp16 means.
 */

/* Bytes of one side record for head dimension d (64, 128 or 256; else 0). */
size_t kvq_nsn_dq_side_bytes(int d);

/*
 * kvq_nsn_dq_quantize -- kvq_nsn_quantize with the side data double-quantized
 * as described above.
 *   x, n_heads, n_tok, layout, codes   as kvq_nsn_quantize (fp16 or bf16 x).
 *   wnorms   device, n_heads * n_tok fp16 (||w_t||), 4-byte aligned.
 *   side     device, n_heads * (n_tok/128) records of kvq_nsn_dq_side_bytes(d)
 *            bytes, 16-byte aligned.
 * Requires a handle without KVQ_QJL (KVQ_EINVAL); fp32 input returns
 * KVQ_EUNSUPPORTED.
 */
int kvq_nsn_dq_quantize(kvq_handle h, const void* x, int dtype, int64_t n_heads, int64_t n_tok, int layout,
                        uint32_t* codes, uint16_t* wnorms, uint8_t* side, void* stream);

/*
 * kvq_nsn_dq_decode_attend -- kvq_nsn_decode_attend over caches written by
 * kvq_nsn_dq_quantize: a stored vector stands for
 *   x_hat = n1/sqrt(d) (w_hat + o_hat_blk),
 * with n1 and o_hat decoded from the side records as above.
 *   k, v      norms hold fp16 ||w|| per token (capacity entries per stream);
 *             codes as usual; capacities multiples of 128.
 *   k_side, v_side  device, per stream capacity/128 side records, stream
 *             (bi, hi) at record (bi * hkv + hi) * capacity/128, 16-byte aligned.
 * Other arguments, workspace and errors as kvq_nsn_decode_attend; every
 * (d, b) is built.
 */
int kvq_nsn_dq_decode_attend(kvq_handle h, const void* q, int dtype, int batch, int hq, int hkv, const kvq_cache* k,
                             const kvq_cache* v, const uint8_t* k_side, const uint8_t* v_side, const int32_t* seq_len,
                             int64_t max_T, float scale, float* logits, float* out, void* workspace, size_t ws_bytes,
                             void* stream);

/* Most tokens a residual window may hold (kvq_decode_desc.window_cap). */
#define KVQ_MAX_WINDOW 256

/* Every argument of a decode call, for kvq_decode_attend_ex. */
typedef struct kvq_decode_desc {
    const void* q;                   /* as kvq_decode_attend */
    int dtype;
    int batch, hq, hkv;
    const kvq_cache* k;
    const kvq_cache* v;
    const uint16_t* k_block_mean;    /* NSN caches (as kvq_nsn_decode_attend), or NULL */
    const uint16_t* v_block_mean;
    const uint16_t* k_window;        /* residual window, fp16 [batch * hkv][window_cap][d], or NULL */
    const uint16_t* v_window;
    int64_t window_cap;              /* 1..KVQ_MAX_WINDOW when a window is given */
    const int32_t* window_len;       /* device, [batch]: tokens in each sequence's window */
    const int32_t* seq_len;          /* device, [batch]: tokens in the packed cache */
    int64_t max_T;
    float scale;
    float* logits;                   /* nullable; row (bi, head) at (bi * hq + head) * logits_ld */
    int64_t logits_ld;               /* 0: max_T (+ window_cap with a window) */
    float* out;
    void* workspace;
    size_t ws_bytes;
    /* NSN caches with double-quantized side data (as kvq_nsn_dq_decode_attend:
     * the norms hold fp16 ||w||), or NULL; not together with block means. */
    const uint8_t* k_side;
    const uint8_t* v_side;
} kvq_decode_desc;

/*
 * kvq_decode_attend_ex -- decode attention over a packed cache, optionally
 * followed by a full-precision residual window (NSNQuant section 4: the newest
 * tokens stay in fp16 until a block of them is flushed into the packed cache),
 * for plain caches, NSN caches with fp16 block means, or NSN caches with
 * double-quantized side records (k_side / v_side).  The softmax runs over the packed tokens [0,
 * seq_len) then the window tokens [0, window_len) of each sequence; window
 * keys and values are used exactly (fp32 arithmetic on the fp16 values).
 * Window logits go to columns max_T + i of the logits rows.  Flushing a full
 * window is kvq_quantize (or kvq_nsn_quantize, kvq_nsn_dq_quantize) of its
 * tokens into the packed arrays at offset seq_len (a multiple of 32; of 128
 * for NSN caches).
 * The workspace size is kvq_decode_workspace's (it covers the window).
 * Errors: as kvq_decode_attend and kvq_nsn_decode_attend; KVQ_EINVAL for a
 * window without all its parts or with window_cap outside 1..KVQ_MAX_WINDOW,
 * for logits_ld too small, and for side records given with block means.
 */
int kvq_decode_attend_ex(kvq_handle h, const kvq_decode_desc* desc, void* stream);

/*
 * kvq_decode_attend_noalloc -- kvq_decode_attend without a caller-provided
 * workspace.  The pages have no counterpart of this call: it exists for
 * callers that cannot allocate device memory at the point where they decode,
 * e.g. a serving engine whose device memory is carved into a fixed pool at
 * start-up and that forbids later cudaMalloc calls, or a plug-in running
 * inside another runtime that owns every allocation.  Instead of a
 * workspace the call uses a scratch array of KVQ_NOALLOC_SCRATCH_BYTES (8 MiB)
 * compiled into the library as a __device__ variable: every GPU that loads
 * the library holds it until the process exits.  The call itself allocates
 * nothing (no cudaMalloc, no cudaFree, no allocating library routine).
 *   Arguments, semantics, outputs and errors are those of kvq_decode_attend
 *   with `workspace`/`ws_bytes` removed.  Sizes whose workspace
 *   (kvq_decode_workspace) exceeds KVQ_NOALLOC_SCRATCH_BYTES are rejected with
 *   KVQ_EINVAL before any launch.
 *   The first call on a device looks up the scratch array's device address
 *   (cudaGetSymbolAddress) with that device current and caches it; make that
 *   first call before any stream capture.
 *   Every call shares the one array and it keeps the last call's contents;
 *   no part of it needs to start at zero (each word read is first written by
 *   the same call).  Calls whose kernels overlap on the GPU (different
 *   streams, or different host threads) race on the array and corrupt each
 *   other's results: serialise them, e.g. on one stream.
 */
int kvq_decode_attend_noalloc(kvq_handle h, const void* q, int dtype, int batch, int hq, int hkv,
                              const kvq_cache* k, const kvq_cache* v, const int32_t* seq_len, int64_t max_T,
                              float scale, float* logits, float* out, void* stream);

/*
 * kvq_probe_wait_timeout -- launch one CTA whose mbarrier wait cannot
 * complete (nothing arrives on it), bounded by `polls` polls (1..2^20), with
 * the same bounded-wait helper every kernel uses.  When the bound runs out
 * the kernel sets KVQ_STATUS_TIMEOUT in the handle's status word and returns,
 * so the next kvq_status reports KVQ_ETIMEOUT and the context stays usable.
 * It exercises the failure path without a fault.  Asynchronous on `stream`.
 */
int kvq_probe_wait_timeout(kvq_handle h, uint32_t polls, void* stream);

/*
 * kvq_status -- synchronise `stream`, read and clear the handle's device
 * status word.  Returns KVQ_OK, KVQ_ENONFINITE or KVQ_ETIMEOUT (the most
 * severe condition seen); *bits (nullable, host) receives the raw
 * KVQ_STATUS_* bits.
 */
int kvq_status(kvq_handle h, void* stream, uint32_t* bits);

/* kvq_last_error -- message of the last failure on this thread ("" if none).
 * The string stays valid until the next kvq_* call on the same thread. */
const char* kvq_last_error(void);

/*
 * kvq_get_constants -- copy the handle's constants to host buffers (any
 * argument may be NULL): signs int8 [d] (+1/-1); S fp16 bit patterns
 * [d][d] row-major; centroids fp32 [2^b] ascending; thresholds fp32
 * [2^b - 1].  Synchronous.
 */
int kvq_get_constants(kvq_handle h, int8_t* signs, uint16_t* S, float* centroids, float* thresholds);

/* kvq_get_info -- d, b, m and flags of a handle (host out-pointers, nullable). */
int kvq_get_info(kvq_handle h, int* d, int* b, int* m, uint32_t* flags);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
