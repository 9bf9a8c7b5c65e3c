/*
 * oq.h -- C ABI of the rotated, quantized linear layer for NVIDIA B200 (sm_100a).
 *
 * The layer (CentriQ: Calibration-Free Quantization of Diffusion Transformers via Exact Mean
 * Centering, §4.2 Eq. 5 and App. B.2 Eq. 9; OrbitQuant PR #25 "Default changes"):
 *
 *     y_t = s_w (.) W_hat_R  Q_a( R (x_t - mean_t 1) )  +  mean_t * w_1  +  b
 *
 *   - mean_t     per-token mean over the d native channels (optional centering, CentriQ §4.2);
 *   - R          RPBH rotation: `rounds` independent rounds, each a gather by a random
 *                permutation, random signs and the orthonormal Sylvester block Hadamard of
 *                size h on consecutive blocks (OrbitQuant PR #25; CentriQ §3, §2);
 *   - Q_a        per-token quantizer: absmax INT8 {-127..127}, absmax INT4 {-7..7}
 *                (CentriQ §3 Eq. 1) or the 16-level N(0,1) Lloyd-Max codebook on x / RMS(x);
 *   - W_hat_R    the weight pre-rotated by the same R (W_R = W R^T) and quantized to INT4
 *                per output channel with scale s_w;
 *   - w_1 = W 1  row sums of the unrotated, unquantized weight, kept in fp32 (CentriQ Eq. 4).
 *
 * Conventions for every call:
 *   - Pointers named *_host are host memory; every other pointer is device memory on the
 *     current CUDA device. The caller owns all buffers and streams; the library owns only
 *     the plan.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Compute calls are
 *     asynchronous on that stream and never synchronize the device.
 *   - Row-major layouts; "ld" arguments are row pitches in elements.
 *   - Argument errors are returned before anything is launched. Launch failures return
 *     OQ_ERR_CUDA. Every device-side wait is bounded: a wait that gives up records a code in
 *     a device error word and the kernel returns; oq_device_status() reads that word.
 *   - oq_last_error() returns a human-readable message for the last failure on the calling
 *     host thread.
 *
 * Data formats:
 *   - activations / weights: bfloat16, row-major [rows, d];
 *   - A8 codes: int8 [T, d];
 *   - 4-bit activation codes: uint8 [rows, d/2], element 2j in bits 0-3 of byte j and
 *     element 2j+1 in bits 4-7; absmax codes are two's-complement nibbles in -7..7,
 *     Lloyd-Max codes are indices 0..15 into the ascending codebook;
 *   - 2-bit activation codes (A2): uint8 [rows, d/4], element 4j + i in bits 2i, 2i + 1 of
 *     byte j, two's complement in -1..1;
 *   - prepared INT4 weights (the GEMM layout): uint8 [d_out, d_in/2] of two's-complement
 *     nibbles in -7..7; every row is split into 16-byte groups, and byte j of group g holds
 *     element 32g + j in bits 0-3 and element 32g + 16 + j in bits 4-7. The GEMM widens a
 *     nibble to the int8 16 n by masking alone;
 *   - per-token scale (alpha_t, or sigma_t for Lloyd-Max), per-token mean, per-channel s_w
 *     and w_1: float32;
 *   - bias: bfloat16 [d_out] or NULL;
 *   - output: bfloat16 [T, d_out] (OQ_OUT_BF16) or raw accumulators [T, d_out] (OQ_OUT_ACC:
 *     int32 for the integer GEMMs, float32 for the Lloyd-Max GEMM).
 *
 * Limits: d % 32 == 0, 32 <= d <= 32768; h a power of two, 1 <= h <= 1024, h | d;
 * rounds in {1, 2}; T >= 0 (T == 0 launches nothing); d_out % 16 == 0; base pointers
 * 16-byte aligned, row pitches multiples of 16 bytes.
 */
#ifndef OQ_H
#define OQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  OQ_OK = 0,
  OQ_ERR_INVALID_ARG = 1,    /* a size, enum or pointer is out of its documented range */
  OQ_ERR_UNSUPPORTED = 2,    /* valid but outside this build (e.g. no sm_100 device)    */
  OQ_ERR_MISALIGNED = 3,     /* a pointer or pitch breaks the 16-byte rule              */
  OQ_ERR_CUDA = 4,           /* a CUDA runtime/driver call failed                       */
  OQ_ERR_DEVICE_TIMEOUT = 5, /* a bounded device-side wait gave up                      */
  OQ_ERR_NOMEM = 6           /* host or device allocation for a plan failed             */
} oq_status;

typedef enum {
  OQ_ACT_INT8_ABSMAX = 0,    /* A8: alpha_t = max|z_t| / 127, codes in -127..127         */
  OQ_ACT_INT4_ABSMAX = 1,    /* A4: alpha_t = max|z_t| / 7,   codes in -7..7             */
  OQ_ACT_INT4_LLOYDMAX = 2,  /* A4: sigma_t = RMS(z_t), nearest of 16 N(0,1) centroids   */
  OQ_ACT_INT4_PERCENTILE = 3, /* A4: percentile range (below), codes clipped to -7..7    */
  OQ_ACT_INT4_LLOYDMAX_WIDTH = 4, /* A4: as LLOYDMAX with the width-d codebook (below)   */
  OQ_ACT_INT8_LLOYDMAX = 5,  /* A8: sigma_t = RMS(z_t), nearest of 256 N(0,1) centroids  */
  OQ_ACT_INT2_PERCENTILE = 6 /* A2: percentile range, codes clipped to -1..1 (below)      */
} oq_act_kind;
/* OQ_ACT_INT8_LLOYDMAX (OrbitQuant PR #25 "Default changes": the 8-bit Lloyd-Max activations
 * that absmax INT8 replaced as the A8 default): codes are uint8 [T, d] indices 0..255 into the
 * 256-level N(0,1) codebook (oq_lloyd_max_codebook_8bit), code = the number of thresholds
 * strictly below z / sigma_t; the GEMM (oq_gemm_w4a8_lloydmax) decodes them to fp16 centroids
 * through a table and runs fp16 x fp16 -> fp32. Limit: d <= 8192. */
/* OQ_ACT_INT4_LLOYDMAX_WIDTH (OrbitQuant PR #25 "Default changes": codebook v3 is one table
 * per width d, solved by Newton's method; CentriQ §2: the codebook is derived from the
 * post-rotation marginal): codes and GEMM as OQ_ACT_INT4_LLOYDMAX, with the 16-level
 * MSE-optimal codebook of the marginal of one coordinate of a width-d token normalised to unit
 * RMS, f_d(y) = c_d (1 - y^2/d)^((d-3)/2) on |y| < sqrt(d) (uniformly random direction; the
 * N(0,1) codebook is its d -> inf limit). See oq_lloyd_max_codebook_width. */
/* OQ_ACT_INT4_PERCENTILE (CentriQ §4.2 "Scale and grid", App. B.3 Tab. 3): the spread of the
 * rotated token is sigma_hat_t = q_rho(|z_t|) / Phi^-1((1 + rho) / 2) with rho = 0.9995, where
 * q_rho is the empirical quantile, linear between the order statistics around position
 * rho (d - 1); alpha_t = max(gamma sigma_hat_t, 1e-10) / 7 with gamma = 2.5591, and
 * codes = clip(round(z / alpha_t), -7, 7). The codes and the GEMM are those of
 * OQ_ACT_INT4_ABSMAX; only the scale differs. Limit: d <= 8192 (the quantile needs the
 * d - floor(rho (d - 1)) <= 6 largest magnitudes, kept per thread). */

/* OQ_ACT_INT2_PERCENTILE (CentriQ Eq. 1 with b = 2, the activation grid of its W4A2 results,
 * App. C.1 Tab. 4; scale of App. B.3 Tab. 3, which is one setting for every b): the range of
 * OQ_ACT_INT4_PERCENTILE, alpha_t = max(gamma sigma_hat_t, 1e-10) / 1, and
 * codes = clip(round(z / alpha_t), -1, 1), i.e. sign(z) where |z| > alpha_t / 2, else 0.
 * Codes are uint8 [T, d/4]: element 4j + i in bits 2i, 2i + 1 of byte j, two's complement
 * (-1 = 0b11). The pages only simulate 2-bit activations (CentriQ §7: no fused kernel supports
 * them yet), so this storage is the library's own. GEMM: oq_gemm_w4a2. Limits: d <= 8192 (as
 * the percentile scale) and d % 64 == 0 (a token's codes are whole 16-byte rows). */

typedef enum {
  OQ_OUT_BF16 = 0,           /* dequantised, rank-1 and bias added, rounded to bf16      */
  OQ_OUT_ACC = 1             /* raw GEMM accumulators, no epilogue (test mode)           */
} oq_out_kind;

typedef struct oq_plan oq_plan; /* opaque, library-owned */

/* ---- status ----------------------------------------------------------------------- */

/* Static string naming a status code. */
const char* oq_status_string(oq_status s);

/* Message describing the last failure on the calling host thread ("" if none). */
const char* oq_last_error(void);

/* Synchronizes the current device, then returns OQ_ERR_DEVICE_TIMEOUT if a kernel recorded
 * a bounded-wait failure since the last clear (its site code in *code_out if non-NULL),
 * OQ_ERR_CUDA if the device reports an error, else OQ_OK. clear != 0 resets the word. */
oq_status oq_device_status(int clear, uint64_t* code_out);

/* ---- policies (host only) ---------------------------------------------------------- */

/* Largest power of two dividing d, capped at 1024 (FLUX.1-schnell-OrbitQuant-W4A4 model card,
 * "Quantization": block size policy largest_power_of_two_dividing_dim). 0 if d <= 0. */
int oq_default_block(int d);

/* 2 if h < 512 else 1 (OrbitQuant PR #25, "Default changes": rotation_rounds "auto"). */
int oq_default_rounds(int h);

/* ---- plan tables (host only, no device needed) ------------------------------------- */

/* Signs (+1/-1) and permutation of RPBH round `round` (0-based) for width d and `seed`.
 * The permutation is a gather: rotated position i reads channel perm_host[i].
 * SplitMix64 in counter form: round r draws signs from key v(seed, 2r) and the
 * permutation from key v(seed, 2r+1), with v(k, i) = mix64(k + (i+1) * 0x9E3779B97F4A7C15);
 * sign i is -1 when bit 63 of v(k_sign, i) is set; perm sorts i by v(k_perm, i), ties by i.
 * signs_host: int8[d], perm_host: int32[d], both caller-owned. */
oq_status oq_rpbh_tables(int d, int round, uint64_t seed, int8_t* signs_host,
                         int32_t* perm_host);

/* 16-level Lloyd-Max codebook for N(0,1), solved by Newton's method on the centroid and
 * midpoint conditions (OrbitQuant PR #25: codebook v3 uses a Newton solver).
 * centroids16_host: double[16] ascending; thresholds15_host: double[15] midpoints. */
oq_status oq_lloyd_max_codebook(double* centroids16_host, double* thresholds15_host);

/* The 256-level N(0,1) Lloyd-Max codebook (OQ_ACT_INT8_LLOYDMAX), solved by Newton's method
 * on the centroid conditions (tridiagonal Jacobian) from the high-resolution point density.
 * centroids256_host: double[256] ascending; thresholds255_host: double[255]. Host only. */
oq_status oq_lloyd_max_codebook_8bit(double* centroids256_host, double* thresholds255_host);

/* The 16-level Lloyd-Max codebook of the width-d marginal f_d (see OQ_ACT_INT4_LLOYDMAX_WIDTH),
 * solved by Newton's method on the centroid and midpoint conditions; cell probabilities by
 * composite Simpson integration of f_d, cell first moments in closed form. Host only.
 * 32 <= d <= 32768, else OQ_ERR_INVALID_ARG. */
oq_status oq_lloyd_max_codebook_width(int d, double* centroids16_host, double* thresholds15_host);

/* ---- plan ------------------------------------------------------------------------------ */

/* Builds the RPBH tables and codebook on the host and uploads the tables (rounds * d
 * uint16 entries, < 128 KiB) to the current device. The plan belongs to that device.
 * center != 0 subtracts the per-token mean before the rotation (CentriQ §4.2). */
oq_status oq_plan_create(oq_plan** out, int d, int h, int rounds, uint64_t seed,
                         int center, oq_act_kind act);

/* Frees the plan and its device tables. NULL is ignored. */
void oq_plan_destroy(oq_plan* plan);

/* Host copies of a plan's RPBH round (same layout as oq_rpbh_tables). */
oq_status oq_plan_get_rpbh(const oq_plan* plan, int round, int8_t* signs_host,
                           int32_t* perm_host);

/* Host copies of the Lloyd-Max codebook a plan quantizes with (OrbitQuant PR #25 "Default
 * changes": codebook v3, one table per width; FLUX.1-schnell-OrbitQuant-W4A4 model card,
 * "Artifact Files": the Lloyd-Max codebooks ship with the rotation metadata as part of the
 * quantized artifact). The table is the one the plan's kernels use: the 16-level N(0,1)
 * codebook for OQ_ACT_INT4_LLOYDMAX, the 16-level width-d codebook for
 * OQ_ACT_INT4_LLOYDMAX_WIDTH, the 256-level N(0,1) codebook for OQ_ACT_INT8_LLOYDMAX.
 *   levels            16 or 256; must be the size of the plan's codebook
 *   centroids_host    double[levels], ascending; thresholds_host double[levels - 1] midpoints
 * OQ_ERR_INVALID_ARG for a NULL argument, a plan whose activation kind uses no codebook
 * (absmax, percentile) or a levels value that is not the plan's. Host only. */
oq_status oq_plan_get_codebook(const oq_plan* plan, int levels, double* centroids_host,
                               double* thresholds_host);

/* ---- compute ----------------------------------------------------------------------- */

/* Fused center + RPBH + per-token scale + quantize (CentriQ §4.2, activation path, and
 * App. B.2, where one prologue centers each token, rotates it and quantizes it with one scale
 * per token; OrbitQuant PR #25 "Runtime work": the pre-rotation runs as a single kernel).
 *   x_bf16       [T, ldx] bf16, ldx >= d, (ldx * 2) % 16 == 0
 *   codes        int8 [T, d] (A8 absmax), uint8 [T, d] (8-bit Lloyd-Max), uint8 [T, d/2]
 *                (A4 kinds) or uint8 [T, d/4] (A2)
 *   scale        float [T]: alpha_t (absmax kinds) or sigma_t (Lloyd-Max)
 *   mean         float [T] per-token mean; required iff the plan centers, else ignored
 *   rotated_f32  float [T, d] normalised rotated (centered) values, or NULL (test output) */
oq_status oq_rotate_quantize(const oq_plan* plan, const void* x_bf16, int64_t T, int64_t ldx,
                             void* codes, float* scale, float* mean, float* rotated_f32,
                             void* stream);

/* Offline weight preparation (CentriQ §3 "Hadamard rotation": W x = (W R^T)(R x); §4.2
 * Eq. 4: w_1 = W 1 in fp32 from the unquantized weight): every row of W goes through the
 * plan's rotation without centering, is quantized to INT4 per output channel
 * (s_w[o] = max|W_R[o,:]| / 7), and w_1[o] = sum_k W[o,k] (fp32, before rotation).
 *   w_bf16    [n_out, ldw] bf16
 *   w_packed  uint8 [n_out, d/2] in the GEMM layout (see "Data formats")
 *   w_scale   float [n_out];  w_rowsum float [n_out] */
oq_status oq_prepare_weights(const oq_plan* plan, const void* w_bf16, int64_t n_out,
                             int64_t ldw, uint8_t* w_packed, float* w_scale,
                             float* w_rowsum, void* stream);

/* Offline preparation of asymmetric grouped INT4 weights (CentriQ §3 Eq. 2; §4.3 "Weight
 * path": groups of g = 64 consecutive columns of the rotated weight W_R, round to nearest
 * from the group minimum and maximum; App. B.2: codes stored as Q - 8; App. B.3 Tab. 3:
 * grid {0..15}, 16-bit scale and zero point). Every row of W goes through the plan's rotation
 * without centering; then per row o and group g:
 *   sigma = fp16(max((max - min) / 15, 2^-14, |min| / 2^15)),  z = fp16(-min / sigma),
 *   Q = clamp(rint(w / sigma + z), 0, 15)        (float32, each step rounded to nearest)
 * (the |min| / 2^15 floor keeps |z| < 2^15 (1 + 2^-11), finite in fp16, for nearly constant
 * groups far from zero)
 * and w_1[o] = sum_k W[o,k] (fp32, before rotation).
 *   plan      d % 64 == 0; its activation kind is not used here
 *   w_bf16    [n_out, ldw] bf16, 16-byte aligned, ldw >= d, (ldw * 2) % 16 == 0
 *   w_packed  uint8 [n_out, d/2] in the GEMM layout, nibble = (Q - 8) two's complement, with
 *             the K order swapped inside every four columns: stored position p holds column
 *             (p & ~3) | ((p & 1) << 1) | ((p >> 1) & 1), i.e. 0, 2, 1, 3 (the order in which
 *             oq_gemm_w4a4_g64 decodes the activation codes)
 *   w_sz      uint32 [d/64][n_out] (group-major): bits 0-15 fp16 sigma, bits 16-31 fp16 z
 *   w_scale   float [n_out]: the per-row scale s_o of §4.3, 1 under round to nearest
 *   w_rowsum  float [n_out]
 * Allocates n_out * d * 4 bytes of stream-ordered scratch (cudaMallocAsync) for the rotated
 * rows; errors as for oq_prepare_weights, OQ_ERR_INVALID_ARG if d % 64 != 0. The fp16 storage
 * bounds the format: a group whose range exceeds 15 * 65504, or whose minimum exceeds 2^15 *
 * 65504 in magnitude (sigma beyond fp16), is not representable and is not detected. */
oq_status oq_prepare_weights_g64(const oq_plan* plan, const void* w_bf16, int64_t n_out,
                                 int64_t ldw, uint8_t* w_packed, uint32_t* w_sz, float* w_scale,
                                 float* w_rowsum, void* stream);

/* W4A8 GEMM with the fused dequant epilogue (CentriQ Eq. 5 / Eq. 9):
 *   acc[t,o] = sum_k a[t,k] * w[o,k]                     (exact int32)
 *   y[t,o]   = bf16( a_scale[t] * w_scale[o] * acc + mean[t] * w_rowsum[o] + bias[o] )
 *   a         int8 [T, d_in]; a_scale float [T]
 *   mean      float [T] or NULL (no rank-1 term; w_rowsum may then be NULL)
 *   w_packed  uint8 [d_out, d_in/2] in the GEMM layout; w_scale float [d_out]
 *   bias_bf16 bf16 [d_out] or NULL
 *   out       bf16 [T, d_out] (OQ_OUT_BF16) or int32 [T, d_out] (OQ_OUT_ACC)
 * For 1 <= T <= 256 with a bf16 result (d_in % 128 == 0) the call runs a split-K cluster GEMM
 * whose int32 partial sums are added exactly in distributed shared memory; the result is the
 * same either way. */
oq_status oq_gemm_w4a8(const int8_t* a, const float* a_scale, const float* mean,
                       const uint8_t* w_packed, const float* w_scale, const float* w_rowsum,
                       const void* bias_bf16, int64_t T, int64_t d_in, int64_t d_out,
                       oq_out_kind out_kind, void* out, void* stream);

/* W4A4 GEMM, same epilogue. kind = OQ_ACT_INT4_ABSMAX or OQ_ACT_INT4_PERCENTILE (integer
 * GEMM, exact int32 accumulators) or OQ_ACT_INT4_LLOYDMAX (codes decoded through the plan's
 * codebook to fp16, fp16 x fp16 -> fp32 GEMM; a_scale holds sigma_t; OQ_OUT_ACC gives
 * float32). `plan` is
 * required for Lloyd-Max (codebook) and ignored otherwise.
 *   a_packed  uint8 [T, d_in/2] */
oq_status oq_gemm_w4a4(const oq_plan* plan, oq_act_kind kind, const uint8_t* a_packed,
                       const float* a_scale, const float* mean, const uint8_t* w_packed,
                       const float* w_scale, const float* w_rowsum, const void* bias_bf16,
                       int64_t T, int64_t d_in, int64_t d_out, oq_out_kind out_kind,
                       void* out, void* stream);

/* W4A4 GEMM against asymmetric grouped weights (oq_prepare_weights_g64), same epilogue:
 *   w_hat[o,k] = fp16(sigma (Q - 8) + fp16(-sigma (z - 8)))   for k in group g = k / 64
 *   acc[t,o]   = sum_k a[t,k] * w_hat[o,k]    (fp16 operands, fp32 accumulation)
 *   y[t,o]     = bf16( a_scale[t] * w_scale[o] * acc + mean[t] * w_rowsum[o] + bias[o] )
 * The zero-point correction of App. B.2 (sigma z' with z' = z - 8, against the group sums of
 * the activation codes) is carried by the dequantized operand; the result is the same sum.
 *   kind      OQ_ACT_INT4_ABSMAX or OQ_ACT_INT4_PERCENTILE; a_packed uint8 [T, d_in/2]
 *   d_in      a multiple of 64; w_sz as written by oq_prepare_weights_g64
 *   out       bf16 [T, d_out] (OQ_OUT_BF16) or float32 acc [T, d_out] (OQ_OUT_ACC)
 *   other arguments as for oq_gemm_w4a8. */
oq_status oq_gemm_w4a4_g64(oq_act_kind kind, const uint8_t* a_packed, const float* a_scale,
                           const float* mean, const uint8_t* w_packed, const uint32_t* w_sz,
                           const float* w_scale, const float* w_rowsum, const void* bias_bf16,
                           int64_t T, int64_t d_in, int64_t d_out, oq_out_kind out_kind,
                           void* out, void* stream);

/* W4A2 GEMM (CentriQ App. C.1: W4A2) for OQ_ACT_INT2_PERCENTILE codes, same epilogue as
 * oq_gemm_w4a8:
 *   acc[t,o] = sum_k a[t,k] * w[o,k]    (a in -1..1, w in -7..7; exact int32)
 *   a_packed  uint8 [T, d_in/4] (four codes per byte, see OQ_ACT_INT2_PERCENTILE)
 *   d_in      a multiple of 64 (else OQ_ERR_INVALID_ARG)
 *   other arguments and out as for oq_gemm_w4a8. */
oq_status oq_gemm_w4a2(const uint8_t* a_packed, const float* a_scale, const float* mean,
                       const uint8_t* w_packed, const float* w_scale, const float* w_rowsum,
                       const void* bias_bf16, int64_t T, int64_t d_in, int64_t d_out,
                       oq_out_kind out_kind, void* out, void* stream);

/* W4A8 GEMM for 8-bit Lloyd-Max codes (OQ_ACT_INT8_LLOYDMAX), same epilogue with
 * a_scale = sigma_t:
 *   acc[t,o] = sum_k c[codes[t,k]] * w[o,k]    (fp16 centroids and weights, fp32 accumulation)
 *   codes     uint8 [T, d_in]; sigma float [T]; `plan` supplies the 256-level codebook and must
 *             have been created with OQ_ACT_INT8_LLOYDMAX (else OQ_ERR_INVALID_ARG)
 *   other arguments and out as for oq_gemm_w4a8 (OQ_OUT_ACC gives float32). */
oq_status oq_gemm_w4a8_lloydmax(const oq_plan* plan, const uint8_t* codes, const float* sigma,
                                const float* mean, const uint8_t* w_packed, const float* w_scale,
                                const float* w_rowsum, const void* bias_bf16, int64_t T,
                                int64_t d_in, int64_t d_out, oq_out_kind out_kind, void* out,
                                void* stream);

/* Bytes of device workspace oq_linear needs for T tokens (codes, scales, means). Where the
 * single launch may run (OQ_ACT_INT8_ABSMAX, OQ_ACT_INT4_ABSMAX and OQ_ACT_INT4_PERCENTILE
 * plans, 1 <= T <= 256) the code region holds one byte per code. */
size_t oq_linear_workspace_bytes(const oq_plan* plan, int64_t T);

/* The whole layer: oq_rotate_quantize into `workspace`, then the GEMM for the plan's
 * activation kind, on one stream. y_bf16 is [T, d_out] bf16. workspace must hold
 * oq_linear_workspace_bytes(plan, T) bytes, 256-byte aligned; it is scratch owned by the
 * caller and overwritten. For INT8 absmax and INT4 (absmax, percentile) plans and
 * 1 <= T <= 256 the call runs as one launch (oq_linear_fused) wherever that path applies; the
 * result, and the scales and means in the workspace, are the same bits either way (INT4 codes
 * are left one per byte by the single launch, two per byte by the two kernels). */
oq_status oq_linear(const oq_plan* plan, const void* x_bf16, int64_t T, int64_t ldx,
                    const uint8_t* w_packed, const float* w_scale, const float* w_rowsum,
                    const void* bias_bf16, int64_t d_out, void* y_bf16, void* workspace,
                    size_t workspace_bytes, void* stream);

/* The whole layer in ONE launch, for small token counts (CentriQ App. B.2: the activation path
 * runs as the prologue of the INT4 GEMM). Same arguments, workspace and result as oq_linear,
 * bit for bit: the kernel first rotates and quantizes the tokens into `workspace` (every CTA takes a
 * share of the token pairs), passes one grid-wide barrier, then runs a split-K GEMM in which a
 * cluster of CTAs shares each 128-channel tile and adds its int32 partial sums through
 * distributed shared memory before the epilogue.
 * INT4 codes are written one two's-complement byte per code (the INT8 layout, values -7..7) and
 * multiplied by the same kind::i8 GEMM; their integer sums are those of oq_gemm_w4a4.
 * Limits: the plan's kind must be OQ_ACT_INT8_ABSMAX, OQ_ACT_INT4_ABSMAX or
 * OQ_ACT_INT4_PERCENTILE, and d <= 8192 with d % 128 == 0;
 * 1 <= T <= 256; the channel tiles' clusters must all fit on the device at once (the launch is
 * cooperative). Outside them it returns OQ_ERR_UNSUPPORTED and launches nothing. */
oq_status oq_linear_fused(const oq_plan* plan, const void* x_bf16, int64_t T, int64_t ldx,
                          const uint8_t* w_packed, const float* w_scale, const float* w_rowsum,
                          const void* bias_bf16, int64_t d_out, void* y_bf16, void* workspace,
                          size_t workspace_bytes, void* stream);

/* oq_linear against asymmetric grouped weights: oq_rotate_quantize into `workspace`, then
 * oq_gemm_w4a4_g64. The plan's activation kind must be OQ_ACT_INT4_ABSMAX or
 * OQ_ACT_INT4_PERCENTILE (else OQ_ERR_INVALID_ARG); workspace as for oq_linear. */
oq_status oq_linear_g64(const oq_plan* plan, const void* x_bf16, int64_t T, int64_t ldx,
                        const uint8_t* w_packed, const uint32_t* w_sz, const float* w_scale,
                        const float* w_rowsum, const void* bias_bf16, int64_t d_out,
                        void* y_bf16, void* workspace, size_t workspace_bytes, void* stream);

/* Size in bytes of the library's static scratch array used by oq_linear_static_scratch. */
#define OQ_STATIC_SCRATCH_BYTES (16u << 20)

/* Allocation-free oq_linear. The pages have no counterpart: this entry point exists for
 * callers that cannot allocate device memory, such as plug-ins running inside a framework
 * that owns all device memory and gives them no allocator, or latency-critical paths that may
 * not call cudaMalloc (it can synchronise the device). It computes exactly what oq_linear
 * computes, with the same arguments except the workspace. Its scratch (codes, scales, means)
 * comes from a 16 MiB array inside the library (OQ_STATIC_SCRATCH_BYTES). Every device that
 * loads the library holds that array until the process exits. The call allocates nothing.
 *   - Limit: oq_linear_workspace_bytes(plan, T) must be <= OQ_STATIC_SCRATCH_BYTES, e.g.
 *     T <= 5447 tokens at d = 3072 with INT8 codes. Larger T returns OQ_ERR_INVALID_ARG
 *     with a message; split the batch or use oq_linear.
 *   - Set-up: the first call on a device looks up the array's device address (with that
 *     device current) and keeps it for the life of the process. Make that first call before
 *     any stream capture. The kept address does not survive cudaDeviceReset (or any other
 *     teardown of the device's primary context): after one, do not call this entry point
 *     again in that process; use oq_linear.
 *   - Sharing: all calls on a device use the same array and leave their contents in it.
 *     Calls whose kernels overlap on the GPU (other streams, other host threads) race on it;
 *     the caller must serialise them. Nothing in the array needs to start at zero. */
oq_status oq_linear_static_scratch(const oq_plan* plan, const void* x_bf16, int64_t T,
                                   int64_t ldx, const uint8_t* w_packed, const float* w_scale,
                                   const float* w_rowsum, const void* bias_bf16, int64_t d_out,
                                   void* y_bf16, void* stream);

/* ---- measurement ------------------------------------------------------------------- */

/* Tensor-core peak loop, the roofline denominator of the GEMMs (the pages have no
 * counterpart; they quote no B200 figure). One CTA pair per two SMs; the pair's leader issues
 * iters x 4 back-to-back tcgen05.mma.cta_group::2 instructions (M = 256, N = 256, 128 bytes of
 * K per group of four) on operand tiles resident in shared memory, into one TMEM accumulator,
 * with no memory traffic. kind 0: kind::i8 (int8 x int8 -> int32, K = 32 per instruction);
 * kind 1: kind::f16 (fp16 x fp16 -> fp32, K = 16); kind 2: kind::i8 with each group of four
 * committed to an mbarrier and waited for before the next is issued, so that its time per
 * group minus kind 0's is the MMA-to-completion latency seen by the issuing thread. One launch
 * performs
 * pairs * iters * 4 * 2 * 256 * 256 * K operations; *pairs_out (may be NULL) receives pairs.
 * Asynchronous on `stream`: time it with events there. iters in [1, 2^16], else
 * OQ_ERR_INVALID_ARG. */
oq_status oq_mma_peak_loop(int kind, int64_t iters, int* pairs_out, void* stream);

/* Inspection hook (host only, no device needed): the word layout a plan of width d, block h
 * and seed gives the two-token rotate-quantize kernel (d <= 8192). Channel j of the
 * interleaved row (both tokens' bf16 values in one 32-bit word) is kept in word word_host[j]
 * (int32[d], caller-owned); bank = word % 32. The layout is an edge colouring chosen so that
 * every warp-wide store of the interleave pass (thread t of a d/32-thread block stores
 * channels 8c + k, c = t + m d/32, m = 0..3, k = 0..7) and every warp-wide round-1 gather
 * (register i of the warp's lanes) touches distinct banks. OQ_ERR_INVALID_ARG if d or h is
 * outside the two-token kernel's range. */
oq_status oq_debug_pair_layout(int d, int h, uint64_t seed, int32_t* word_host);

/* Test hook for the bounded waits: launches one block that waits on an mbarrier nothing
 * will arrive on, for at most timeout_ns, then records a timeout and returns. The next
 * oq_device_status() reports OQ_ERR_DEVICE_TIMEOUT. The GPU stays usable. */
oq_status oq_debug_wait_timeout(uint64_t timeout_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* OQ_H */
