/*
 * kvq.h -- C ABI of the B200 (sm_100a) fused KV-cache rotate-and-quantize
 * library (libkvq.so).
 *
 * The operation, per KV vector x of length D (one layer / K-or-V / kv-head /
 * token row of an fp16 cache):
 *
 *   y = H_D diag(s) (lambda . x) / sqrt(D)          (smooth scale + SRHT)
 *   S_j = fp16(max_{i in group j} |y_i| / 7)         (per-group abs-max)
 *   q_i = clamp(rint(y_i * (1/S_j)), -8, 7)          (signed int4)
 *   two codes per byte, even element in the low nibble
 *
 * and the inverse  x_hat = (diag(s) H_D (q . S) / sqrt(D)) / lambda.
 *
 * Sources: "When Quantization Is Free: An int4 KV Cache That Outruns fp16 on
 * Apple Silicon" (arXiv 2605.05699) -- Abstract (one fused kernel: sign-
 * randomised transform + per-channel lambda + per-group abs-max + int4
 * nibble pack; SRFT and SRHT equivalent in quality) and the technical
 * summary on gist.science, Methodologie 1-3 (fixed random sign vector;
 * kernel steps load & sign-multiply, transform, lambda rescale, per-group
 * absolute-max reduction, round to signed int4, pack two int4 per byte;
 * groups of 16).  The order "smooth scale, Hadamard transform, quantize /
 * dequantize, inverse transform, unscale" follows "The Kernel That Finally
 * Did Something" (VeloxQuant-MLX blog), section "The kernel toggle".
 *
 * Exact arithmetic contract (what makes results reproducible bit for bit):
 *   - x_i * lambda_i is rounded to fp32 before any addition (no FMA);
 *   - the unnormalised transform runs radix-2 butterflies with ascending
 *     half-width h = 1, 2, ..., D/2, each output one fp32 a+b or a-b;
 *   - y_i = v_i * c with c the fp32 value nearest 1/sqrt(D);
 *   - S_j = fp16 round-to-nearest-even of the fp32 IEEE quotient max|y|/7,
 *     saturated to 65504; a zero S_j gives zero codes;
 *   - q_i = rint(y_i * r_j), r_j = fp32 IEEE reciprocal of S_j, round half
 *     to even, saturated to [-8, 7];
 *   - inverse: u_i = q_i * S_j (exact), the same transform, z_i = u_i * c,
 *     out_i = fp16_rne((s_i z_i) * (1/lambda_i)), 1/lambda_i an fp32 IEEE
 *     reciprocal.
 *
 * Memory: every pointer is DEVICE memory owned by the caller.  The library
 * allocates nothing, keeps no state between calls except a per-device cache
 * of launch limits, one per-device fault word (below) and the static 8 MiB
 * scratch array of kvq_attention_decode_static (one per device, shared by
 * every call of that entry point; see there), and never synchronises.
 * Calls are asynchronous on `stream` (a cudaStream_t; NULL means the legacy
 * default stream) and launch on the calling thread's current device, which
 * must own the buffers and the stream.
 *
 * Errors: a failed precondition returns a negative kvq_status before any
 * launch, and nothing is written.  A launch failure returns
 * KVQ_ERR_LAUNCH.  Faults during execution surface, as usual in CUDA, at
 * the caller's next synchronising runtime call.  The kernels stage data with
 * asynchronous bulk copies and wait for them on shared-memory barriers; every
 * such wait is bounded, and a block that gives up sets the device's fault
 * word and returns with its outputs incomplete (kvq_fault_status).
 */
#ifndef KVQ_H
#define KVQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KVQ_OK = 0,
    KVQ_ERR_NULL = -1,    /* a required pointer is NULL                    */
    KVQ_ERR_ALIGN = -2,   /* a pointer violates its alignment requirement  */
    KVQ_ERR_DIM = -3,     /* D is not 64, 128 or 256                        */
    KVQ_ERR_GROUP = -4,   /* group is not a power of two in [16, D]         */
    KVQ_ERR_COUNT = -5,   /* n_vec < 0 or n_vec > 2^31 - 256                */
    KVQ_ERR_LAUNCH = -6   /* the kernel launch failed (see kvq_last_cuda_error) */
} kvq_status;

/*
 * kvq_quantize -- rotate, quantise and pack n_vec vectors.
 *
 *   x       [in]  fp16 (IEEE binary16 bits) [n_vec][D], row-major, contiguous.
 *                 16-byte aligned.  Finite values (NaN/Inf are not supported).
 *   lambda  [in]  float32 [D]  per-channel smooth scale; 4-byte aligned;
 *                 finite and non-zero.
 *   signs   [in]  int8 [D]  the random sign vector; each entry +1 or -1 (any
 *                 negative value is read as -1, anything else as +1).
 *   n_vec         number of vectors (rows), 0 <= n_vec <= 2^31 - 256 (the copy
 *                 engine's row coordinates are 32-bit); 0 is a no-op
 *                 returning KVQ_OK; larger counts return KVQ_ERR_COUNT
 *                 (split the call).
 *   D             head dimension: 64, 128 or 256.
 *   group         group size G: a power of two with 16 <= G <= D.
 *   packed  [out] uint8 [n_vec][D/2]: code 2b in the low nibble of byte b,
 *                 code 2b+1 in the high nibble, 4-bit two's complement.
 *                 16-byte aligned.
 *   scales  [out] fp16 bits [n_vec][D/G]; 2-byte aligned.
 *   stream        cudaStream_t to launch on.
 *
 * `x` must not overlap `packed` or `scales`.
 */
int kvq_quantize(const uint16_t *x, const float *lambda, const int8_t *signs,
                 int64_t n_vec, int D, int group,
                 uint8_t *packed, uint16_t *scales, void *stream);

/*
 * kvq_quantize_rows -- kvq_quantize with a row map: vector r of x is encoded
 * into row row_idx[r] of packed / scales, whose rows 0 .. cache_rows-1
 * belong to the caller (e.g. one new token per sequence appended into its
 * slot of a decode cache).  Rows not named in row_idx are left untouched.
 *
 *   row_idx     [in] int64 [n_vec], device memory, 8-byte aligned.  An index
 *               outside [0, cache_rows) is skipped (nothing is written for
 *               that vector) and sets bit 2 of the fault word.  Two vectors
 *               with the same index race; either result may remain.
 *   cache_rows  number of rows of packed / scales (>= 0).
 *   Other arguments as for kvq_quantize.
 */
int kvq_quantize_rows(const uint16_t *x, const float *lambda, const int8_t *signs,
                      int64_t n_vec, int D, int group,
                      const int64_t *row_idx, int64_t cache_rows,
                      uint8_t *packed, uint16_t *scales, void *stream);

/*
 * kvq_dequantize -- unpack, rescale, inverse-rotate and un-scale n_vec
 * vectors.  Same layouts and conventions as kvq_quantize.
 *
 *   packed  [in]  uint8 [n_vec][D/2]; 16-byte aligned.
 *   scales  [in]  fp16 bits [n_vec][D/G]; 2-byte aligned.
 *   lambda, signs, n_vec, D, group: as for kvq_quantize (same values that
 *                 produced the codes).
 *   x_out   [out] fp16 bits [n_vec][D]; 16-byte aligned; must not overlap
 *                 the inputs.
 */
int kvq_dequantize(const uint8_t *packed, const uint16_t *scales,
                   const float *lambda, const int8_t *signs,
                   int64_t n_vec, int D, int group,
                   uint16_t *x_out, void *stream);

/*
 * kvq_dequantize_tc -- kvq_dequantize with the Walsh-Hadamard transform's
 * in-group factor on the tensor cores, bit-identical to kvq_dequantize.
 * H_D = (H_(D/G) (x) I_G)(I_(D/G) (x) H_G): inside a group u = q S stays an
 * exact multiple of S, so H_G q is a sum of small integers that a tensor-core
 * product with fp16 codes and a +-1 matrix (fp32 accumulation) gets exactly;
 * the stages that cross groups run as fp32 butterflies in the contract's
 * order.  (The pages' "16x16 matrix-multiply alignment", technical summary,
 * Methodologie 1, "Redenering"; a variant kept beside the butterfly kernel.)
 * Same arguments, layouts and results as kvq_dequantize; D must be 128 (else
 * KVQ_ERR_DIM) and group 16, 32 or 64 (else KVQ_ERR_GROUP).
 */
int kvq_dequantize_tc(const uint8_t *packed, const uint16_t *scales,
                      const float *lambda, const int8_t *signs,
                      int64_t n_vec, int D, int group,
                      uint16_t *x_out, void *stream);

/*
 * kvq_roundtrip -- x_hat = kvq_dequantize(kvq_quantize(x)) in one pass over
 * x (the quantise-then-dequantise shape used to simulate the cache's error
 * on the fly), bit-identical to the two calls back to back.
 *
 *   x, lambda, signs, n_vec, D, group: as for kvq_quantize.
 *   x_hat   [out] fp16 bits [n_vec][D]; 16-byte aligned; must not overlap x.
 *   packed, scales [out, optional] the codes and scales as kvq_quantize
 *                  writes them; pass both or neither (NULL).
 */
int kvq_roundtrip(const uint16_t *x, const float *lambda, const int8_t *signs,
                  int64_t n_vec, int D, int group, uint16_t *x_hat,
                  uint8_t *packed, uint16_t *scales, void *stream);

/*
 * kvq_quantize_ex / kvq_dequantize_ex -- the codec with format options.
 *   flags bit 0 (KVQ_LAMBDA_AFTER)  0: lambda before the rotation, y =
 *                    R (lambda . x) (as kvq_quantize); 1: after it, y =
 *                    lambda . (R x), the order of "When Quantization Is
 *                    Free", technical summary, Methodologie 2 (transform of
 *                    diag(s) x, then the per-channel lambda rescale).  The
 *                    inverse divides by lambda (fp32 multiply by IEEE
 *                    1/lambda) before its transform instead of after.
 *   flags bit 1 (KVQ_SRFT)  R = H diag(s) / sqrt(D) (0), or the SRFT (1):
 *                    pack(F diag(s) .), F the unitary DFT (same summary,
 *                    Methodologie 1), computed as a length-D/2 complex FFT
 *                    in radix-2 Stockham stages with the Hermitian unpacking
 *                    y0 = X_0, y1 = X_D/2, (y_2k, y_2k+1) = sqrt(2) (Re, Im)
 *                    X_k, all divided by sqrt(D).
 *   bits          4: int4 codes packed two per byte as kvq_quantize, S =
 *                    fp16(max|y| / 7); 8: one int8 code per byte (two's
 *                    complement), S = fp16(max|y| / 127), codes in [-128, 127].
 *   lambda        n_lambda tables of D floats, fp32, 4-byte aligned; vector r
 *                 uses table (r / lambda_rows) % n_lambda (per-(layer, head)
 *                 smoothing: for a [layers][K,V][heads][T][D] cache,
 *                 lambda_rows = T and n_lambda = layers * 2 * heads).  With
 *                 n_lambda > 1, lambda_rows must be a multiple of 32.
 *   codes         uint8 [n_vec][D/2] (bits 4) or [n_vec][D] (bits 8),
 *                 16-byte aligned.  Other arguments as for kvq_quantize /
 *                 kvq_dequantize.
 * D must be 128 (else KVQ_ERR_DIM); group in {16, 32, 64}, bits in {4, 8} and
 * no other flag bits (else KVQ_ERR_GROUP); n_vec, lambda_rows, n_lambda out of
 * range -> KVQ_ERR_COUNT.  Results are bit-identical to the oracle's definition
 * of each option; bits = 4, flags = 0 and one table reproduce kvq_quantize /
 * kvq_dequantize exactly.
 */
#define KVQ_LAMBDA_AFTER 1
#define KVQ_SRFT 2
int kvq_quantize_ex(const uint16_t *x, const float *lambda, const int8_t *signs,
                    int64_t n_vec, int D, int group, int bits, int flags,
                    int64_t lambda_rows, int n_lambda, uint8_t *codes,
                    uint16_t *scales, void *stream);
int kvq_dequantize_ex(const uint8_t *codes, const uint16_t *scales,
                      const float *lambda, const int8_t *signs, int64_t n_vec,
                      int D, int group, int bits, int flags,
                      int64_t lambda_rows, int n_lambda, uint16_t *x_out,
                      void *stream);

/*
 * kvq_attention_decode -- one decode step of attention over the int4 cache:
 * for every sequence b and query head h,
 *     o[b][h] = sum_t p_t V_t,  p = softmax_t(sm_scale <q[b][h], K_t>),
 * over the keys t < seq_len[b] of KV head h / (Hq / Hkv) (grouped-query
 * attention), where K_t and V_t are the rows kvq_dequantize would rebuild
 * from the codes, but never rounded to fp16 nor written anywhere.  The
 * operation is the fused group-quantised attention of "The Kernel That
 * Finally Did Something -- And Didn't Quite Agree With Itself" (VeloxQuant-MLX
 * blog), "Fused group-affine (KIVI-style) attention", taken to the rotated
 * domain of "When Quantization Is Free" (Methodologie 1): the query is
 * rotated once, q~ = H diag(s_K)(q / lambda_K)/sqrt(D), scores are
 * <q~, codes * S>, the values are summed in the rotated domain and rotated
 * back once per head.  An empty context (seq_len[b] = 0) gives zeros.
 *
 *   q         [in]  fp16 bits [B][Hq][D]; 16-byte aligned.
 *   k_packed, v_packed  [in] uint8 [B][Hkv][T][D/2] (kvq_quantize rows, one
 *                   cache row per (sequence, KV head, position)); 16-byte
 *                   aligned.
 *   k_scales, v_scales  [in] fp16 bits [B][Hkv][T][D/group]; 16-byte aligned.
 *   seq_len   [in]  int32 [B], device memory, 4-byte aligned; each in [0, T]
 *                   (a value outside is clamped and sets bit 3 of the fault
 *                   word).
 *   lambda_k, signs_k, lambda_v, signs_v  [in] the parameters the K and V
 *                   rows were quantised with (fp32 [D], 4-byte aligned;
 *                   int8 [D] with values +-1).
 *   B, Hq, Hkv, T  sequences, query heads, KV heads, cache positions:
 *                   B >= 0, Hkv >= 1, Hq a multiple of Hkv with Hq / Hkv <= 8,
 *                   T >= 0 a multiple of 16, B * Hkv * T < 2^40 cache rows,
 *                   < 2^31 at D = 256 (whose code tiles arrive by tensor
 *                   copies with 32-bit row coordinates; 2^31 rows of K codes
 *                   alone are 256 GiB) (else KVQ_ERR_COUNT).
 *   D, group  D in {64, 128, 256} (else KVQ_ERR_DIM); group in
 *                   {16, 32, 64, 128}, group <= D (else KVQ_ERR_GROUP).
 *   sm_scale  softmax scale, finite (usually 1/sqrt(D)).
 *   out       [out] fp16 bits [B][Hq][D]; 16-byte aligned; must not overlap
 *                   the inputs.
 *   workspace, workspace_bytes  optional device scratch for splitting the
 *                   key axis when B * Hkv is too small to fill the GPU; give
 *                   at least kvq_attention_workspace_bytes() bytes, 16-byte
 *                   aligned.  With less (or NULL) the call runs unsplit: same
 *                   result up to fp32 summation order, possibly slower.  The
 *                   library allocates nothing.
 *   stream    cudaStream_t (NULL: legacy default stream); asynchronous.
 * B = 0 is a no-op.  Preconditions are checked in the order shape, NULL,
 * alignment.
 */
int kvq_attention_decode(const uint16_t *q, const uint8_t *k_packed,
                         const uint16_t *k_scales, const uint8_t *v_packed,
                         const uint16_t *v_scales, const int32_t *seq_len,
                         const float *lambda_k, const int8_t *signs_k,
                         const float *lambda_v, const int8_t *signs_v,
                         int B, int Hq, int Hkv, int T, int D, int group,
                         float sm_scale, uint16_t *out, void *workspace,
                         int64_t workspace_bytes, void *stream);

/*
 * kvq_attention_decode_ex -- kvq_attention_decode over a cache written by
 * kvq_quantize_ex with int4 codes (bits 4): `flags` is the cache's format,
 * bit 0 (KVQ_LAMBDA_AFTER) lambda after the rotation, bit 1 (KVQ_SRFT) the
 * SRFT rotation ("When Quantization Is Free", technical summary,
 * Methodologie 1-2: the paper's own cache is KVQ_SRFT | KVQ_LAMBDA_AFTER).
 * The rows are rebuilt as (diag(s) R^T (codes . S)) / lambda with lambda
 * before the rotation, diag(s) R^T ((codes . S) / lambda) with lambda after
 * it, R^T the inverse Walsh-Hadamard or SRFT rotation; the query is rotated
 * once to match and the rotated-domain output rotated back once per head.
 * One lambda table per K and per V (lambda_rows = all rows).  Other flag bits
 * -> KVQ_ERR_GROUP; other arguments, checks and results as for
 * kvq_attention_decode, which is this call with flags = 0.  The SRFT
 * rotations run inside the kernels (a warp-wide real FFT per row, roots
 * computed on the device): no call copies tables from the host, so every
 * call may sit inside a stream capture.
 */
int kvq_attention_decode_ex(const uint16_t *q, const uint8_t *k_packed,
                            const uint16_t *k_scales, const uint8_t *v_packed,
                            const uint16_t *v_scales, const int32_t *seq_len,
                            const float *lambda_k, const int8_t *signs_k,
                            const float *lambda_v, const int8_t *signs_v,
                            int B, int Hq, int Hkv, int T, int D, int group, int flags,
                            float sm_scale, uint16_t *out, void *workspace,
                            int64_t workspace_bytes, void *stream);

/*
 * kvq_attention_workspace_bytes -- bytes of workspace kvq_attention_decode
 * uses for these shapes on the current device (0: it does not split), or -1
 * if the shapes are invalid.  Host-only; launches nothing.
 */
int64_t kvq_attention_workspace_bytes(int B, int Hq, int Hkv, int T, int D, int group);

/*
 * kvq_attention_decode_static -- kvq_attention_decode without a caller
 * workspace and without any allocation: the key-split scratch is a static
 * 8 MiB device array inside the library (one per device, held by every GPU
 * that loads the library until the process exits).  The pages have no
 * counterpart of this entry point; it exists for callers that cannot hand out
 * device memory (a caller inside a stream capture or a callback that may not
 * allocate, or one whose allocator is owned by a host framework).  Same
 * arguments, results and checks as kvq_attention_decode; returns
 * KVQ_ERR_COUNT when the shapes need more split scratch than 8 MiB
 * (kvq_attention_workspace_bytes() > 8 MiB).  The first call on a device that
 * needs the scratch looks its device address up (cudaGetSymbolAddress, with
 * that device current) and caches it: make that first call before any stream
 * capture, and do not use the entry point across a cudaDeviceReset, which
 * invalidates the cached address.  Calls that overlap in time share the
 * scratch and race: serialise them (one stream, or events between streams and
 * host threads).
 */
int kvq_attention_decode_static(const uint16_t *q, const uint8_t *k_packed,
                                const uint16_t *k_scales, const uint8_t *v_packed,
                                const uint16_t *v_scales, const int32_t *seq_len,
                                const float *lambda_k, const int8_t *signs_k,
                                const float *lambda_v, const int8_t *signs_v,
                                int B, int Hq, int Hkv, int T, int D, int group,
                                float sm_scale, uint16_t *out, void *stream);

/*
 * kvq_fault_status -- the current device's fault word: 0 when every bounded
 * wait of every kernel so far completed; bit 0 set when a quantize,
 * dequantize (base or _ex) or attention warp gave up waiting for its bulk
 * copies (its outputs are then incomplete); bit 1 set by kvq_selftest_wait_timeout; bit 2 set when
 * kvq_quantize_rows skipped an out-of-range row index; bit 3 set when
 * kvq_attention_decode met a sequence length outside [0, T].  Non-zero `clear`
 * resets the word.  Synchronous (it copies the word to the host, which waits
 * for prior work on the device's legacy default stream).  Returns -1 if the
 * word cannot be read.
 */
int kvq_fault_status(int clear);

/*
 * kvq_selftest_wait_timeout -- launches one block that waits, at most `limit`
 * polls, on a shared-memory barrier that nothing completes, and then takes
 * the same give-up path as the real kernels (sets bit 1 of the fault word and
 * returns).  It exists to test that path; it touches no caller memory.
 * Returns KVQ_OK or KVQ_ERR_LAUNCH.
 */
int kvq_selftest_wait_timeout(uint32_t limit, void *stream);

/*
 * kvq_selftest_rcp_f16 -- writes the reciprocal the quantisers use for a group
 * scale S (r = 1/S, an approximate reciprocal refined by one Newton step) for
 * every positive finite fp16 value: out[i] = r(S) for the fp16 S whose bit
 * pattern is i + 1, i = 0 .. 31742.  It exists so that a test can check that r
 * is the IEEE fp32 quotient 1/S for every scale the codec can store.
 *   out     [out] float32 [31743], device memory, 4-byte aligned.
 * Returns KVQ_OK, KVQ_ERR_NULL, KVQ_ERR_ALIGN or KVQ_ERR_LAUNCH; asynchronous
 * on `stream`.
 */
int kvq_selftest_rcp_f16(float *out, void *stream);

/* Human-readable name of a kvq_status value (static storage). */
const char *kvq_status_string(int status);

/* The cudaError_t value behind the calling thread's last KVQ_ERR_LAUNCH
 * (0 if none). */
int kvq_last_cuda_error(void);

/* Library ABI version: (major << 16) | minor. */
int kvq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
