/*
 * kvrq -- online vector quantization of KV-cache vectors on NVIDIA B200 (sm_100a).
 *
 * C ABI of libkvrq.so. Every hot-path call launches hand-written CUDA kernels
 * asynchronously on the given stream and returns a status; nothing here
 * allocates device memory, and no call synchronises the device except
 * kvrq_device_status().
 *
 * Sources of the method (cited by page title and section):
 *   [RQ]  "TurboQuant + RotorQuant" (README of the RotorQuant repository),
 *         sections "How TurboQuant Works", "How RotorQuant Works",
 *         "FMA Count (d=128)", "Codebook Calibration Fix",
 *         "Post-Prefill Quantization", "The Fused CUDA Kernel",
 *         "Non-Commutative Algebra Bug Fix", "Triton Kernels".
 *   [TQB] "TurboQuant 论文解读" (TurboQuant paper walkthrough), sections
 *         "随机旋转（Lemma 1）", "Beta 分布", "MSE 标量量化（Theorem 1）",
 *         "QJL 内积无偏估计（Theorem 2）", "简单复现 demo".
 *   [TQA] arXiv 2504.19874 summary page, section "方法" (Algorithms 1 and 2).
 *   [PQ]  "TurboQuant и PolarQuant: математика квантизации KV-кэша в LLM",
 *         paragraph on building codebooks with Lloyd's algorithm; the
 *         attention formula in "Проблема KV-кэша в трансформерах".
 *
 * Conventions shared by all calls
 * -------------------------------
 *  - stream: a cudaStream_t passed as void* (NULL = legacy default stream).
 *  - Device pointers are caller-owned and must stay valid until the stream
 *    reaches the call. Vector/tile pointers must be 16-byte aligned; row
 *    strides (ld*) are in elements (words for packed codes) and must make
 *    every row start 16-byte aligned unless a call says otherwise.
 *  - Packed codes: per row one little-endian bit stream, code j in bits
 *    [j*b, j*b+b) (LSB first), cut into 32-bit words; a row holds
 *    kvrq_packed_words(n_codes, b) words and unused high bits are zero.
 *  - QJL signs: bit j of a row is 1 for sign +1 and 0 for -1 (sign(0) = +1),
 *    m/32 words per row.
 *  - n == 0 is a no-op returning KVRQ_OK (after argument checks); the one
 *    exception is kv_attention_packed with no tokens (KVRQ_EINVAL).
 *  - Arguments are validated on the host before any launch; a bad argument
 *    returns KVRQ_EINVAL / KVRQ_EUNSUPPORTED and launches nothing. A failed
 *    launch returns KVRQ_ECUDA. kvrq_last_error_string() explains the last
 *    non-OK status of the calling thread.
 *  - Kernels that wait on barriers bound every wait; on time-out they record
 *    KVRQ_ETIMEOUT in a device status word, which kvrq_device_status() reads.
 */
#ifndef KVRQ_H
#define KVRQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KVRQ_OK = 0,
  KVRQ_EINVAL = 1,       /* bad pointer, size, stride or alignment */
  KVRQ_EUNSUPPORTED = 2, /* valid but not implemented (e.g. bits outside 1..4) */
  KVRQ_ECUDA = 3,        /* a CUDA runtime/driver call failed */
  KVRQ_ENOCONV = 4,      /* Lloyd-Max did not converge within max_iter */
  KVRQ_ETIMEOUT = 5,     /* a bounded device-side wait ran out */
  KVRQ_ENOMEM = 6,       /* host memory could not be allocated (the call changed nothing) */
  KVRQ_ECHECKSUM = 7     /* a parameter file's contents do not match its checksum */
} kvrq_status;

typedef enum { KVRQ_F32 = 0, KVRQ_F16 = 1, KVRQ_BF16 = 2 } kvrq_dtype;

typedef enum { KVRQ_RQ_MSE = 0, KVRQ_TQ_MSE = 1, KVRQ_TQ_PROD = 2 } kvrq_method;

/* Version string of the library. */
const char* kvrq_version(void);

/* Message for the last non-OK status returned on this thread ("" if none). */
const char* kvrq_last_error_string(void);

/* Reads (and clears) the device status word written by bounded waits.
 * Synchronises `stream`. Returns KVRQ_OK, KVRQ_ETIMEOUT or KVRQ_ECUDA. */
kvrq_status kvrq_device_status(void* stream);

/* ===================================================================== setup
 * Host-only, float64, deterministic functions of their arguments. No CUDA
 * call is made. Output arrays are caller-owned host memory.
 */

/* Number of 32-bit words holding n_codes codes of `bits` bits: ceil(n*b/32). */
int64_t kvrq_packed_words(int64_t n_codes, int bits);

/* RotorQuant group count G = ceil(d/3) [RQ "How RotorQuant Works": d=128 -> 43]. */
int kvrq_rq_groups(int d);

/* Lloyd-Max codebook for one coordinate of a uniform unit vector in R^d, density
 * f(x) ~ (1-x^2)^((d-3)/2) on [-1,1] [TQB "Beta 分布", "MSE 标量量化（Theorem 1）"],
 * iterated as in [PQ]: boundaries at midpoints, centroids at conditional means,
 * until max |change| < tol or max_iter iterations. Use d_eff = d for RotorQuant
 * too [RQ "Codebook Calibration Fix"]. Centroids are returned ascending and
 * exactly symmetric (c[i] = -c[K-1-i]); boundaries[k] = (c[k]+c[k+1])/2.
 *   d >= 2, 1 <= bits <= 8, tol > 0, max_iter >= 1.
 *   centroids: [2^bits] out. boundaries: [2^bits - 1] out (may be NULL).
 *   iterations: out (may be NULL).
 * Returns KVRQ_ENOCONV if not converged (outputs then hold the last iterate). */
kvrq_status tq_codebook_init(int d, int bits, double tol, int max_iter, double* centroids,
                             double* boundaries, int* iterations);

/* PolarQuant angle codebook of one level ["TurboQuant и PolarQuant: математика
 * квантизации KV-кэша в LLM", "Полярное преобразование", "Шаг 3: построение кодовых
 * книг"]: level-1 angles (of coordinate pairs) are uniform on [0, 2 pi); an angle of
 * level l >= 2 pairs the norms of two k = 2^(l-1)-dimensional sub-vectors and has
 * density Gamma(k) / (2^(k-2) Gamma(k/2)^2) sin^(k-1)(2 theta) on [0, pi/2]
 * (sin^2 theta ~ Beta(k/2, k/2)). Lloyd iteration as for tq_codebook_init, from an
 * even grid; level >= 2 centroids are returned exactly symmetric about pi/4.
 *   1 <= level <= 20, 1 <= bits <= 8, tol > 0, max_iter >= 1.
 *   centroids: [2^bits] out, ascending. boundaries: [2^bits - 1] out (may be NULL).
 *   iterations: out (may be NULL).
 * Returns KVRQ_ENOCONV if not converged (outputs then hold the last iterate). */
kvrq_status pq_angle_codebook_init(int level, int bits, double tol, int max_iter, double* centroids,
                                   double* boundaries, int* iterations);

/* G = ceil(d/3) random unit rotors (s, b12, b13, b23), row-major [G][4]
 * [RQ "How RotorQuant Works": R = [s,0,0,0,b12,b13,b23,0]]: 4 standard normals
 * per group from the counter-based stream `seed` (splitmix64 + Box-Muller, see
 * below), divided by their norm (uniform on the unit 3-sphere). d >= 1. */
kvrq_status rq_rotors_init(int d, uint64_t seed, double* rotors);

/* Random orthogonal Pi [d][d] row-major [TQB "随机旋转（Lemma 1）"]: Householder
 * QR of the Gaussian matrix A[i][j] = normal(i*d+j) of stream `seed`, then
 * Pi = Q diag(sign(diag R)) (unique, Haar distributed). 1 <= d <= 16384. */
kvrq_status tq_rotation_init(int d, uint64_t seed, double* pi);

/* QJL projection T [m][d] row-major, T[i][j] = normal(i*d+j) of stream `seed`
 * [TQB "QJL 内积无偏估计（Theorem 2）": Gaussian S]. The sketch uses S = T Pi,
 * which is again i.i.d. N(0,1); the kernels then work in rotated coordinates. */
kvrq_status qjl_matrix_init(int m, int d, uint64_t seed, double* T);

/* Random streams: normal number i of stream s is taken from splitmix64 outputs
 * 2j, 2j+1 (j = i/2; output k = mix64(s + (k+1)*0x9E3779B97F4A7C15)), turned
 * into uniforms ((out>>11)+1)*2^-53 and into two normals by Box-Muller
 * (cos for even i, sin for odd i). Exposed for tests: out[k] = normal(first+k). */
kvrq_status kvrq_normals(uint64_t seed, int64_t first, int64_t count, double* out);

/* ================================================================ RotorQuant
 * [RQ "How RotorQuant Works", "The Fused CUDA Kernel", "Codebook Calibration
 * Fix"]: u = x/||x|| (norm stored separately), u zero-padded to 3G coordinates,
 * each group g rotated by the sandwich v' = R_g v R_g~ (computed as the exact
 * 3x3 matrix of that sandwich), each of the 3G rotated coordinates replaced by
 * the index of its nearest centroid (ties -> lower index), codes packed.
 * Dequantization looks the centroids up, applies the inverse sandwich
 * R_g~ v R_g, drops coordinates >= d and multiplies by the norm.
 *
 *   x       [n][ldx] device, dtype xdtype, row-major, first d entries used.
 *   rotors  [G][4] fp32 device (s, b12, b13, b23).
 *   centroids [2^bits] fp32 device, ascending.
 *   codes   [n][ldc] uint32 device, ldc >= kvrq_packed_words(3G, bits).
 *   norms   [n] fp32 device (||x||, 0 for a zero row).
 *   xhat    [n][ldo] device, dtype of x (dequantize: odtype).
 *   1 <= bits <= 4, d >= 2. Fast paths: d = 128 (and d = 256 for fp16/bf16) with 16-byte
 *   aligned rows, one thread per row; other d with 16-byte aligned rows stream whole rows
 *   through shared memory, a warp per row.
 */
kvrq_status rq_quantize(void* stream, const void* x, kvrq_dtype xdtype, int64_t n, int d, int64_t ldx,
                        const float* rotors, const float* centroids, int bits, uint32_t* codes,
                        int64_t ldc, float* norms);

kvrq_status rq_dequantize(void* stream, const uint32_t* codes, int64_t ldc, const float* norms, int64_t n,
                          int d, const float* rotors, const float* centroids, int bits, void* xhat,
                          kvrq_dtype odtype, int64_t ldo);

/* One fused launch of quantize and dequantize [RQ "Triton Kernel Speed": the
 * whole embed -> rotor -> quantize -> unrotor -> extract pipeline in a single
 * launch]: writes codes, norms and xhat (same dtype as x). codes and norms may
 * be NULL (xhat only), xhat may not. */
kvrq_status rq_quantize_dequantize(void* stream, const void* x, kvrq_dtype xdtype, int64_t n, int d,
                                   int64_t ldx, const float* rotors, const float* centroids, int bits,
                                   uint32_t* codes, int64_t ldc, float* norms, void* xhat, int64_t ldo);

/* RotorQuant fused roundtrip of rows in HOST memory ["TurboQuant + RotorQuant", "Post-Prefill
 * Quantization" (a prefill cache quantized in bulk) and "Triton Kernel Speed" (one fused launch per
 * block of vectors)]: the rows are copied to the device in chunks, each chunk is quantized and
 * dequantized there by rq_quantize_dequantize, and its codes, norms and x_hat are copied back; the
 * copy-in of one chunk, the kernel of the previous one and the copy-out of the one before run at
 * once, on three streams the library creates per device. The call is ordered after the work queued
 * on `stream` before it (and after the copy-outs of earlier calls of this function on the device),
 * work queued on `stream` after it waits for its last copy-out, and it returns without waiting.
 *   x      [n][ldx] host rows (fp32, fp16 or bf16), xhat [n][ldo] host rows of the same dtype;
 *   codes  [n][ldc] host uint32 (may be NULL), norms [n] host fp32 (may be NULL);
 *   rotors, centroids: device arrays as for rq_quantize_dequantize.
 *   workspace: device memory, 256-byte aligned, of workspace_bytes >= kvrq_host_workspace_bytes(d,
 *   bits, xdtype, 32); the call takes the largest chunk (32 rows times a power of two) whose three
 *   slots fit, at most the input rounded up to 32 rows. Host arrays should be page-locked
 *   (cudaHostAlloc, cudaHostRegister): pageable memory gives the same results with the copies
 *   serialised by the driver. Nothing is allocated by the call.
 *   KVRQ_EINVAL: NULL pointers, ldx, ldo < d, ldc below the code words of a row, a misaligned or
 *   too small workspace; these are checked before anything is queued. KVRQ_ECUDA: a copy, event
 *   or launch failed; copies and kernels queued before the failure may still run, so the caller
 *   synchronizes the device before reusing the buffers. */
kvrq_status rq_quantize_dequantize_host(void* stream, const void* x, kvrq_dtype xdtype, int64_t n, int d,
                                        int64_t ldx, const float* rotors, const float* centroids, int bits,
                                        uint32_t* codes, int64_t ldc, float* norms, void* xhat, int64_t ldo,
                                        void* workspace, size_t workspace_bytes);

/* Device workspace bytes rq_quantize_dequantize_host needs for chunks of chunk_rows rows (rounded up
 * to a multiple of 32; at least 32): three slots of x and x_hat rows padded to 16 bytes, code words
 * and norms. 0 for arguments the call rejects. */
size_t kvrq_host_workspace_bytes(int d, int bits, kvrq_dtype dtype, int64_t chunk_rows);

/* RotorQuant in the pages' four-grade storage layout [RQ "Parameter Efficiency"
 * (rotors plus four grade codebooks), "FMA Count (d=128)" table (172 stored
 * indices per vector, 3.7x at 3 bits), "The Fused CUDA Kernel" (a grade-1 input
 * gives vector and trivector outputs)]: per group the stored indices are the
 * three vector components of R v R~ and its trivector component, code k = 4g + i
 * (i = 0, 1, 2: e1, e2, e3; i = 3: e123), 4G codes per row (172 at d = 128).
 * The trivector component of a unit-rotor sandwich is identically zero and is
 * stored as the code of exactly 0, 2^(bits-1) - 1 (ties to the lower index); the
 * inverse sandwich maps a pseudoscalar to itself, so dequantization ignores it
 * and x_hat equals that of the three-code layout. Vector and trivector share the
 * one Lloyd-Max codebook (the pages define no other).
 *   Arguments as rq_quantize / rq_dequantize / rq_quantize_dequantize, with
 *   ldc >= kvrq_packed_words(4G, bits) (17 words at d = 128, 3 bits).
 *   d = 128 only, rows 16-byte aligned (one dtype for the fused call); other
 *   shapes return KVRQ_EUNSUPPORTED before any launch. */
kvrq_status rq4_quantize(void* stream, const void* x, kvrq_dtype xdtype, int64_t n, int d, int64_t ldx,
                         const float* rotors, const float* centroids, int bits, uint32_t* codes, int64_t ldc,
                         float* norms);

kvrq_status rq4_dequantize(void* stream, const uint32_t* codes, int64_t ldc, const float* norms, int64_t n, int d,
                           const float* rotors, const float* centroids, int bits, void* xhat, kvrq_dtype odtype,
                           int64_t ldo);

kvrq_status rq4_quantize_dequantize(void* stream, const void* x, kvrq_dtype xdtype, int64_t n, int d, int64_t ldx,
                                    const float* rotors, const float* centroids, int bits, uint32_t* codes,
                                    int64_t ldc, float* norms, void* xhat, int64_t ldo);


/* ================================================================ PolarQuant
 * ["TurboQuant и PolarQuant: математика квантизации KV-кэша в LLM": "Шаг 1:
 * предобусловливание" (a fixed random rotation), "Полярное преобразование" (level 1
 * pairs consecutive coordinates (a, b) into a radius and an angle atan2(b, a) in
 * [0, 2 pi); every further level pairs consecutive radii of the level below, angles
 * in [0, pi/2]), "Шаг 3: построение кодовых книг" (one Lloyd-Max codebook per level,
 * nearest centroid), "Степень сжатия" (d = 128: four levels of 4, 2, 2, 2 bits and the
 * 8 last radii as 16-bit floats, 496 bits per vector)]:
 *   y = Pi x, the polar transform of y, every angle replaced by the index of its
 *   nearest centroid (ties to the lower index; a zero pair has angle 0), the 8
 *   level-4 radii rounded to fp16; x_hat = Pi^T y_hat, y_hat rebuilt from the
 *   codes and the 16-bit radii (r cos c_hat, r sin c_hat, level by level).
 *   x, x_hat: [n][ldx], [n][ldo] fp16 or bf16 (xdtype / odtype), rows 16-byte aligned.
 *   pi: [128][128] row-major in the vector type, 16-byte aligned (Pi of tq_rotation_init).
 *   centroids: [28] fp32 device: level 1 (16; the Lloyd-Max codebook of the uniform
 *     angle, (2i + 1) pi/16, whose boundaries are the multiples of pi/8: the kernel
 *     decides level-1 codes against those boundaries), then 4 for each of levels 2,
 *     3, 4 ascending (pq_angle_codebook_init(level, 2)); the boundaries of levels
 *     2..4 are the midpoints of neighbouring centroids.
 *   codes: [n][ldc] uint32, ldc >= 16: words 0..7 the 64 level-1 codes (4 bits,
 *     LSB first), 8..9 the 32 level-2 codes, 10 the 16 level-3 codes, 11 the 8
 *     level-4 codes (bits 0..15; bits 16..31 zero), 12..15 the 8 level-4 radii as
 *     fp16 pairs (radius 2c in the low half of word 12 + c).
 *   d = 128 only; other shapes and dtypes return KVRQ_EUNSUPPORTED before any
 *   launch. The rotations run on the tensor cores (16-bit operands, fp32
 *   accumulation). pq_quantize_dequantize: codes may be NULL (x_hat only). */
kvrq_status pq_quantize_dequantize(void* stream, const void* x, kvrq_dtype xdtype, int64_t n, int d, int64_t ldx,
                                   const void* pi, const float* centroids, uint32_t* codes, int64_t ldc, void* xhat,
                                   int64_t ldo);

kvrq_status pq_dequantize(void* stream, const uint32_t* codes, int64_t ldc, int64_t n, int d, const void* pi,
                          const float* centroids, void* xhat, kvrq_dtype odtype, int64_t ldo);


/* ================================================================ TurboQuant
 * [TQA "方法" Algorithm 1; TQB "随机旋转（Lemma 1）"]: u = x/||x||, y = Pi u,
 * each y_i replaced by its nearest Lloyd-Max centroid (codebook for d, ties to
 * the lower index), codes packed; dequantize x_hat = ||x|| Pi^T c_hat.
 * [TQA Algorithm 2; TQB "QJL 内积无偏估计（Theorem 2）"; RQ "How TurboQuant
 * Works"] (prod, b bits): (b-1)-bit codes as above, rotated residual
 * r = y - c_hat, gamma = ||r||, signs s = sign(T (256 r)) with the operand
 * rounded to fp16 (S = T Pi is the pages' Gaussian projection; sign(0) = +1),
 * x_hat = ||x|| Pi^T (c_hat + sqrt(pi/2)/m gamma T^T s).
 *
 * Two tensor-core paths, chosen by d and the vector type:
 *  - d = m = 128, fp16 or bf16 vectors: one launch per call, Pi (and T) kept in
 *    shared memory;
 *  - d a multiple of 128 (fp16/bf16: d >= 256; fp32: any such d, d = 128
 *    included), m = d: a tiled contraction that streams Pi / T, two launches
 *    for the fused quantize + dequantize and for each prod call; the prod calls
 *    pass the rotated residual (or the QJL-corrected centroids) between their
 *    two launches through `workspace`, in blocks of rows.
 * x (and x_hat) fp32, fp16 or bf16; Pi [d][d] row-major in the vector type
 * (fp16 for fp32 vectors, which are split into fp16 hi + lo parts on the
 * tensor cores); T [m][d] row-major fp16. Pi, T, x, x_hat and workspace
 * 16-byte aligned, rows of x / x_hat 16-byte aligned. centroids: [2^b] (mse)
 * or [2^(b-1)] (prod) fp32, ascending and symmetric. codes [n][ldc] uint32
 * with ldc >= kvrq_packed_words(d, b or b-1); signs [n][lds] uint32,
 * lds >= m/32; norms, gammas [n] fp32. Other shapes return KVRQ_EUNSUPPORTED.
 */
kvrq_status tq_quantize_mse(void* stream, const void* x, kvrq_dtype xdtype, int64_t n, int d, int64_t ldx,
                            const void* pi, const float* centroids, int bits, uint32_t* codes, int64_t ldc,
                            float* norms);

/* Fused quantize + dequantize. At d = 128 (fp16/bf16) one launch with two MMAs
 * per tile, and codes and norms may be NULL; on the tiled path the dequantize
 * launch reads the codes and norms the quantize launch wrote, so both are
 * required. */
kvrq_status tq_quantize_dequantize_mse(void* stream, const void* x, kvrq_dtype xdtype, int64_t n, int d, int64_t ldx,
                                       const void* pi, const float* centroids, int bits, uint32_t* codes,
                                       int64_t ldc, float* norms, void* xhat, int64_t ldo);

/* Bytes of workspace the tiled prod path uses for `rows` rows at dimension d:
 * rows * (4 d + 4 d / 128). A call given workspace_bytes processes its rows in
 * blocks of floor(workspace_bytes / kvrq_tq_workspace_bytes(1, d) / 128) * 128
 * rows (at least 128 rows must fit). The d = 128 fp16/bf16 path needs none. */
size_t kvrq_tq_workspace_bytes(int64_t rows, int d);

/* TurboQuant-prod quantize, b = bits in 2..5 total bits per coordinate.
 * workspace: device buffer owned by the caller (NULL / 0 where none is needed),
 * overwritten; calls sharing a workspace must be ordered on one stream. */
kvrq_status tq_quantize_prod(void* stream, const void* x, kvrq_dtype xdtype, int64_t n, int d, int64_t ldx,
                             const void* pi, const uint16_t* T, int m, const float* centroids, int bits,
                             uint32_t* codes, int64_t ldc, uint32_t* signs, int64_t lds, float* gammas,
                             float* norms, void* workspace, size_t workspace_bytes);

/* tq_quantize_prod without a workspace argument: the tiled path runs its row
 * blocks through a static 8 MiB device array of the library (address taken
 * once per device at set-up), so the call allocates nothing and takes no
 * buffer beyond its outputs. The pages have no counterpart of this call; it
 * exists for callers that may not allocate. Same arguments and results as
 * tq_quantize_prod; returns KVRQ_EUNSUPPORTED when one 128-row block does not
 * fit the array (128 * kvrq_tq_workspace_bytes(1, d) > 8 MiB, i.e. d = 16384).
 * Nothing in the array has to start at zero. Calls that overlap in time on one
 * device (other streams, other host threads) share the array and race: order
 * them on one stream. */
kvrq_status tq_quantize_prod_noalloc(void* stream, const void* x, kvrq_dtype xdtype, int64_t n, int d, int64_t ldx,
                                     const void* pi, const uint16_t* T, int m, const float* centroids, int bits,
                                     uint32_t* codes, int64_t ldc, uint32_t* signs, int64_t lds, float* gammas,
                                     float* norms);

/* Dequantize mse (signs == NULL; bits = b) or prod (signs != NULL; bits = b
 * total; workspace as for tq_quantize_prod). */
kvrq_status tq_dequantize(void* stream, const uint32_t* codes, int64_t ldc, const uint32_t* signs, int64_t lds,
                          const float* gammas, const float* norms, int64_t n, int d, int m, int bits,
                          const void* pi, const uint16_t* T, const float* centroids, void* xhat, kvrq_dtype odtype,
                          int64_t ldo, void* workspace, size_t workspace_bytes);

/* The QJL map on its own [TQB "QJL 内积无偏估计（Theorem 2）"; RQ "How
 * TurboQuant Works"]: for each row r of the [n][ldr] matrix, signs = sign(T r)
 * (bit j = 1 for T_j . r >= 0) and gammas = ||r||. r fp32, fp16 or bf16; T [m][d]
 * row-major in the type of r (fp16 for fp32 r, which is split into hi + lo
 * parts). d a multiple of 64, m a multiple of 128; signs [n][lds] uint32 with
 * lds >= m/32; gammas [n] at stride ldn. */
kvrq_status qjl_sketch(void* stream, const void* r, kvrq_dtype rdtype, int64_t n, int d, int64_t ldr, const void* T,
                       int m, uint32_t* signs, int64_t lds, float* gammas, int64_t ldn);

/* ================================================================ scores from packed keys
 * [TQB "随机旋转（Lemma 1）": rotate the query once instead of every key;
 * RQ "How TurboQuant Works": <q,k> ~ <q,k_mse> + ||r|| sqrt(pi/2)/m <S q, sign(S r)>;
 * RQ "When to Use Which": Q K^T straight from the compressed indices]
 *   score[h][g][t] = ||k|| * ( <q', c_hat(k)> + [prod] sqrt(pi/2)/m * gamma(k) * <T q', s(k)> )
 * with q' = Pi q (TurboQuant) or the per-group rotor sandwich of the zero-padded q
 * (RotorQuant, 3G coordinates); equal to <q, x_hat(k)>.
 *   q: [n_heads][group][ldq] (dtype qdtype), grouped-query layout: query row
 *      (h, g) reads KV head h. n_heads counts every (layer, batch, KV head).
 *   keys of head h, token t: codes + h*codes_head_stride + t*ldc (words),
 *      signs + h*signs_head_stride + t*lds (prod), norms/gammas + h*tok_head_stride + t.
 *   method KVRQ_RQ_MSE (rotors [43][4]), KVRQ_TQ_MSE or KVRQ_TQ_PROD (pi [d][d] of
 *      pi_dtype fp16/bf16, T [m][d] fp16 for prod); bits = the quantizer's total bits
 *      (prod stores bits-1); centroids: the stored codes' codebook.
 *   scores: fp32 [(h*group + g)*ld_scores + t].
 * d = 128 (m = d); group <= 64 (prod: <= 32). Scores use fp16 operands on the
 * tensor cores with fp32 accumulation. */
kvrq_status kv_score_packed(void* stream, kvrq_method method, const void* q, kvrq_dtype qdtype, int64_t ldq,
                            int64_t n_heads, int group, int d, int bits, int m, const uint32_t* codes, int64_t ldc,
                            int64_t codes_head_stride, const uint32_t* signs, int64_t lds, int64_t signs_head_stride,
                            const float* norms, const float* gammas, int64_t tok_head_stride, int64_t n_tokens,
                            const float* rotors, const void* pi, kvrq_dtype pi_dtype, const uint16_t* T,
                            const float* centroids, float* scores, int64_t ld_scores);

/* Parameter files: the seed-derived parameters of one configuration (d, bits, m,
 * seed) written once and read back, verified ["TurboQuant 论文解读", "简单复现 demo";
 * "TurboQuant + RotorQuant", "How RotorQuant Works", "Codebook Calibration Fix": the
 * rotation, the Gaussian projection, the rotors and the codebook are fixed functions
 * of the seed and the sizes]. The file is a magic line "KVRQ-PARAMS 1", a one-line
 * JSON header (d, bits, m, seed, the array lengths and "fnv1a64", the FNV-1a 64-bit
 * hash of the payload in hex) and the float64 arrays little-endian: rotors [G][4]
 * (rq_rotors_init, seed + 1), pi [d][d] (tq_rotation_init, seed + 2), T [m][d]
 * (qjl_matrix_init, seed + 3), centroids [2^bits] (tq_codebook_init, tol 1e-13).
 *   export: 2 <= d <= 16384, 1 <= bits <= 8, 1 <= m <= 16384; KVRQ_EINVAL if the
 *     file cannot be written.
 *   import: the file must hold exactly that (d, bits, m) (else KVRQ_EINVAL, as for a
 *     missing, malformed or wrong-length file); payload bytes that do not hash to the
 *     header's checksum return KVRQ_ECHECKSUM and write nothing. Output arrays may
 *     be NULL (skipped); seed receives the file's seed (may be NULL). Host only. */
kvrq_status kvrq_params_export(const char* path, int d, int bits, int m, uint64_t seed);
kvrq_status kvrq_params_import(const char* path, int d, int bits, int m, uint64_t* seed, double* rotors, double* pi,
                               double* T, double* centroids);

/* Time-out path of the device waits: every wait of a kernel on a copy or a
 * tensor-core product polls a bounded number of times, then records KVRQ_ETIMEOUT
 * in the device status word (read and cleared by kvrq_device_status), waits at the
 * default limit for its own copies and products still in flight, frees its tensor
 * memory and returns (its outputs are then incomplete). kvrq_set_wait_limit sets
 * the polls of the packed-score kernel's main-loop waits and of the tensor-core
 * attention kernel's tile-copy waits for the calls that follow in this process
 * (negative: the default, 2^24 polls), so a test can make a wait
 * run out with no fault: with 0 those waits give up without polling (a single poll
 * may itself block until a copy lands). */
void kvrq_set_wait_limit(int64_t polls);

/* Test hook of the host failure path: the next `count` host allocations made by
 * the library's entry points (parameter setup work vectors, page-manager tables)
 * fail as if memory were exhausted; each such call returns KVRQ_ENOMEM and changes
 * nothing. count <= 0 disarms the hook. No device memory is involved. */
void kvrq_test_fail_allocations(int count);

/* ================================================================ paged KV cache
 * ["TurboQuant + RotorQuant", "Post-Prefill Quantization": the prefill cache is
 * quantized in bulk, then one new key and value per decode step; with many sequences
 * of different lengths the packed rows live in pages of a pool]
 * A paged cache keeps, for every pool head p = layer * kv_heads + k (one per layer
 * and KV head), its packed rows in slots of a pool: codes + p * codes_pool_stride +
 * slot * ldc, signs + p * signs_pool_stride + slot * lds, norms / gammas (and value
 * norms) + p * tok_pool_stride + slot. Sequence s owns pages of page_tokens slots
 * listed by its block table (the kvrq_pages_* bookkeeping below hands them out):
 * token t < seq_lens[s] sits at slot page_tokens * block_tables[s * ld_table +
 * t / page_tokens] + t % page_tokens. Head h of a call is (layer, sequence, KV
 * head), h = (layer * n_seqs + s) * kv_heads + k, so n_heads is a multiple of n_seqs
 * x kv_heads. block_tables and seq_lens are device int32 arrays the kernels read;
 * the caller keeps every slot they name inside the pools. */
typedef struct kvrq_paged {
  const int32_t* block_tables; /* device [n_seqs][ld_table] */
  int64_t ld_table;            /* >= ceil(max_tokens / page_tokens) */
  const int32_t* seq_lens;     /* device [n_seqs], tokens of each sequence (<= max_tokens) */
  int32_t page_tokens;         /* slots per page, >= 1 (a power of two >= 16 keeps bulk copies) */
  int32_t n_seqs;
  int32_t kv_heads;
} kvrq_paged;

/* kv_score_packed over a paged cache: scores [(h*group + g)*ld_scores + t] for
 * t < seq_lens[s] of head h's sequence (others untouched); max_tokens bounds the
 * sequence lengths (it sizes the launch, ld_scores >= max_tokens). Other arguments
 * as kv_score_packed, the head strides stepping pool heads. */
kvrq_status kv_score_packed_paged(void* stream, kvrq_method method, const void* q, kvrq_dtype qdtype, int64_t ldq,
                                  int64_t n_heads, int group, int d, int bits, int m, const uint32_t* codes,
                                  int64_t ldc, int64_t codes_pool_stride, const uint32_t* signs, int64_t lds,
                                  int64_t signs_pool_stride, const float* norms, const float* gammas,
                                  int64_t tok_pool_stride, const kvrq_paged* paged, int64_t max_tokens,
                                  const float* rotors, const void* pi, kvrq_dtype pi_dtype, const uint16_t* T,
                                  const float* centroids, float* scores, int64_t ld_scores);

/* kv_attention_packed over a paged cache (keys and values share the slots): every
 * query row of head h attends over the seq_lens[s] tokens of its sequence (a
 * sequence of no tokens gives a zero output). Runs where
 * kvrq_attention_uses_tensor_cores is 1; other configurations return
 * KVRQ_EUNSUPPORTED. workspace: kvrq_attention_workspace_bytes(n_heads, group,
 * max_tokens) bytes. Other arguments as kv_attention_packed, the head strides
 * stepping pool heads. */
kvrq_status kv_attention_packed_paged(void* stream, kvrq_method k_method, const void* q, kvrq_dtype qdtype,
                                      int64_t ldq, int64_t n_heads, int group, int d, float scale, int k_bits, int m,
                                      const uint32_t* k_codes, int64_t ldk, int64_t k_pool_stride,
                                      const uint32_t* k_signs, int64_t lds, int64_t s_pool_stride,
                                      const float* k_norms, const float* k_gammas, const float* k_rotors,
                                      const void* pi, kvrq_dtype pi_dtype, const uint16_t* T,
                                      const float* k_centroids, const uint32_t* v_codes, int64_t ldv,
                                      int64_t v_pool_stride, const float* v_norms, int v_bits,
                                      const float* v_rotors, const float* v_centroids, int64_t tok_pool_stride,
                                      const kvrq_paged* paged, int64_t max_tokens, void* out, kvrq_dtype odtype,
                                      int64_t ldo, void* workspace, size_t workspace_bytes);

/* Quantizes row r of x into pool row dst_rows[r] (device int64 [n_rows], e.g.
 * p * slots_per_pool + slot of the new token): codes + dst_rows[r] * ldc, signs +
 * dst_rows[r] * lds, norms / gammas + dst_rows[r] * ldn, in one launch; the decode
 * step of a paged cache. method and parameters as kv_cache_append; d = 128 with
 * 16-byte aligned rows (TurboQuant: fp16 or bf16), else KVRQ_EUNSUPPORTED. */
kvrq_status kv_cache_append_rows(void* stream, kvrq_method method, const void* x, kvrq_dtype xdtype, int64_t n_rows,
                                 int d, int64_t ldx, int bits, const float* rotors, const void* pi, const uint16_t* T,
                                 int m, const float* centroids, const int64_t* dst_rows, uint32_t* codes,
                                 int64_t ldc, uint32_t* signs, int64_t lds, float* norms, float* gammas,
                                 int64_t ldn);

/* ================================================================ decode-step append
 * [RQ "Post-Prefill Quantization": each decode step quantizes the new key (and
 * value) for storage] Quantizes one new vector per cache row (a row = one
 * (layer, batch, KV head)) straight into its slot of a packed cache, in one
 * launch: row r of x goes to codes + r*codes_row_stride (words), signs +
 * r*signs_row_stride, norms/gammas + r*norm_row_stride. The caller passes the
 * cache pointers already advanced to the slot (e.g. codes + slot*W). method
 * selects rq_quantize, tq_quantize_mse or tq_quantize_prod (same argument
 * rules); unused parameters may be NULL. */
kvrq_status kv_cache_append(void* stream, kvrq_method method, const void* x, kvrq_dtype xdtype, int64_t n_rows,
                            int d, int64_t ldx, int bits, const float* rotors, const void* pi, const uint16_t* T, int m,
                            const float* centroids, uint32_t* codes, int64_t codes_row_stride, uint32_t* signs,
                            int64_t signs_row_stride, float* norms, float* gammas, int64_t norm_row_stride);

/* ================================================================ decode attention from packed keys and values
 * ["TurboQuant и PolarQuant: математика квантизации KV-кэша в LLM", "Проблема
 * KV-кэша в трансформерах": attention is softmax(q K^T / sqrt(d)) V; "TurboQuant +
 * RotorQuant", "When to Use Which": for speed, attention is computed from the
 * compressed indices instead of a decompressed cache]
 *   out[h][g] = sum_t softmax_t(scale * <q_(h,g), k_hat_t>) * v_hat_t
 * for every query row (h, g) over the first n_tokens tokens of KV head h. k_hat:
 * keys dequantized by k_method (the logits are the scores of kv_score_packed);
 * v_hat: RotorQuant-dequantized values. Nothing is dequantized into memory.
 *   q: [n_heads][group][ldq] of qdtype, as for kv_score_packed.
 *   keys: k_codes + h*k_head_stride + t*ldk (words), k_signs + h*s_head_stride +
 *     t*lds (prod), k_norms/k_gammas + h*tok_head_stride + t; parameters k_rotors
 *     (RotorQuant keys, [43][4]) or pi (pi_dtype fp16/bf16) and T (prod, [m][d]
 *     fp16); k_bits = the key quantizer's total bits (prod stores k_bits - 1);
 *     k_centroids: the stored key codes' codebook.
 *   values: RotorQuant codes v_codes + h*v_head_stride + t*ldv (3G = 129 codes of
 *     v_bits each per row), v_norms + h*tok_head_stride + t, v_rotors [43][4],
 *     v_centroids [2^v_bits].
 *   scale: multiplies the logits (1/sqrt(d) for standard attention).
 *   out: [(h*group + g)*ldo + i], i < d, of odtype.
 *   workspace: device memory owned by the caller, at least
 *     kvrq_attention_workspace_bytes(n_heads, group, n_tokens) bytes, 16-byte
 *     aligned, overwritten; calls sharing it must be ordered on one stream.
 * d = 128 (m = d); group in 1..16; k_bits 1..4 (prod 2..4); v_bits 1..4;
 * n_heads <= 65535. n_heads = 0 is a no-op; n_tokens = 0 with n_heads > 0 is
 * KVRQ_EINVAL (a softmax over no tokens is undefined). Where
 * kvrq_attention_uses_tensor_cores is 1 both contractions run on the tensor cores
 * (fp16 operands, fp32 accumulation), else in fp32 on the CUDA cores; three
 * launches either way (query rotation, per-chunk online softmax and value sums,
 * chunk merge with one inverse sandwich per query row). */
size_t kvrq_attention_workspace_bytes(int64_t n_heads, int group, int64_t n_tokens);

kvrq_status kv_attention_packed(void* stream, kvrq_method k_method, const void* q, kvrq_dtype qdtype, int64_t ldq,
                                int64_t n_heads, int group, int d, float scale, int k_bits, int m,
                                const uint32_t* k_codes, int64_t ldk, int64_t k_head_stride, const uint32_t* k_signs,
                                int64_t lds, int64_t s_head_stride, const float* k_norms, const float* k_gammas,
                                const float* k_rotors, const void* pi, kvrq_dtype pi_dtype, const uint16_t* T,
                                const float* k_centroids, const uint32_t* v_codes, int64_t ldv, int64_t v_head_stride,
                                const float* v_norms, int v_bits, const float* v_rotors, const float* v_centroids,
                                int64_t tok_head_stride, int64_t n_tokens, void* out, kvrq_dtype odtype, int64_t ldo,
                                void* workspace, size_t workspace_bytes);

/* Which kernel kv_attention_packed runs for keys of k_method (k_bits total
 * bits), values of v_bits bits and `group` query rows per KV head: 1 when both
 * contractions run on the tensor cores (fp16 operands: decoded centroids, +-1
 * signs, rotated queries and softmax weights, fp32 accumulation; outputs within
 * 1e-2 of the row's largest |output|), 0 for the fp32 CUDA-core kernel (1e-3).
 * Tensor cores take: TurboQuant-prod keys of 3 or 4 bits with group <= 8,
 * TurboQuant-mse keys of 2..4 bits and RotorQuant keys of 2 or 3 bits with group
 * <= 16, all with 3-bit values. Host only; no device is touched. */
int kvrq_attention_uses_tensor_cores(kvrq_method k_method, int k_bits, int v_bits, int group);

/* ================================================================ paged cache bookkeeping (host)
 * ["TurboQuant + RotorQuant", "Post-Prefill Quantization": the prefill cache is
 * quantized in bulk once, then one new key/value per decode step.] A pool of
 * n_pages pages of page_tokens token slots each, and per sequence the block table
 * of the pages its tokens occupy in order: logical token t of a sequence is pool slot
 * page_tokens * table[t / page_tokens] + t % page_tokens. The packed rows (codes,
 * signs, norms, gammas) are caller-owned device arrays indexed by slot; these calls
 * only keep the tables (host memory, no CUDA call, thread-safe per pool).
 *   create: n_pages in 1..2^31-1, page_tokens >= 1; destroy(NULL) is a no-op.
 *   add_seq: a new empty sequence; its id is never reused by this pool.
 *   append: reserves n_tokens more slots at the end of the sequence (new pages from
 *     the free list as needed); *first_token (may be NULL) = its previous length.
 *     KVRQ_EINVAL and nothing reserved if the free pages do not suffice.
 *   slots: slots[k] = pool slot of logical token first + k (all below the length).
 *   block_table: the sequence's pages in order into pages[capacity] (KVRQ_EINVAL if
 *     capacity is too small; *n_pages and *n_tokens, either may be NULL, are set
 *     anyway).
 *   free_seq: returns the sequence's pages to the free list and forgets the id.
 * Unknown sequence ids and NULL pools return KVRQ_EINVAL. */
typedef struct kvrq_pages kvrq_pages;
kvrq_status kvrq_pages_create(int64_t n_pages, int page_tokens, kvrq_pages** out);
void kvrq_pages_destroy(kvrq_pages* pages);
kvrq_status kvrq_pages_add_seq(kvrq_pages* pages, int64_t* seq_id);
kvrq_status kvrq_pages_append(kvrq_pages* pages, int64_t seq_id, int64_t n_tokens, int64_t* first_token);
kvrq_status kvrq_pages_slots(kvrq_pages* pages, int64_t seq_id, int64_t first, int64_t count, int64_t* slots);
kvrq_status kvrq_pages_block_table(kvrq_pages* pages, int64_t seq_id, int32_t* table, int64_t capacity,
                                   int64_t* n_pages, int64_t* n_tokens);
kvrq_status kvrq_pages_free_seq(kvrq_pages* pages, int64_t seq_id);
kvrq_status kvrq_pages_stats(kvrq_pages* pages, int64_t* free_pages, int64_t* n_seqs);

#ifdef __cplusplus
}
#endif

#endif /* KVRQ_H */
