/*
 * quip.h — C ABI of libquip: incoherence-processed LDLQ for one linear layer
 * on one NVIDIA B200 (sm_100a).
 *
 * The method is QuIP ("QuIP: 2-Bit Quantization of Large Language Models With
 * Guarantees", arXiv 2307.13304) with the randomized Hadamard incoherence of
 * QuIP# ("QuIP#: Even Better LLM Quantization with Hadamard Incoherence and
 * Lattice Codebooks", arXiv 2402.04396, abstract).  For W in R^{m x n} and
 * calibration activations X in R^{N x n} the library computes, all on the GPU:
 *
 *   H   = X^T X / N                           (QuIP, adaptive-rounding section)
 *   H  += alpha * mean(diag H) * I            (QuIP, Experiments, "Methods.")
 *   W~  = U W V^T,  H~ = V H V^T              (QuIP, incoherence processing)
 *   H~  = (I + Ů) D (I + Ů)^T, Ů strictly upper         (LDL factorisation)
 *   per row: lo = min W~_i,  s = (max W~_i - lo) / (2^b - 1)
 *   for k:  a_k = W~_k + sum_{j<k} (W~_j - W^_j) Ů_jk,  c_k = Q(a_k),
 *           W^_k = lo + s c_k                               (LDLQ)
 *   W^  = U^T W~^ V                           (QuIP, incoherence post-processing)
 *
 * with U (m side) and V (n side) each a randomized Hadamard transform
 * H_d diag(s) / sqrt(d) (d a power of two) or a Kronecker product A (x) B of
 * two Haar-random orthogonal matrices (QuIP, Introduction).
 *
 * Conventions for every entry point
 *  - Matrices are row-major.  "device" pointers are CUDA global memory of
 *    the current device; "host" pointers are ordinary CPU memory.
 *  - The caller owns every buffer it passes; the library never frees or
 *    keeps a caller pointer after the call returns.  The library owns only
 *    quip_transform objects (created / destroyed below).
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls only
 *    enqueue work on it and return before the work finishes, unless stated.
 *  - Argument and shape errors are returned synchronously before anything
 *    is launched.  Errors found on the device (a non-positive LDL pivot, a
 *    non-finite value, a bounded wait that ran out) set a library status
 *    word that quip_sync_status() returns.
 *  - Workspace: entry points that take (ws, ws_bytes) need at least the
 *    bytes quip_workspace_size() reports for the same arguments, device
 *    memory, 256-byte aligned; the contents on entry are irrelevant.
 */
#ifndef QUIP_H_
#define QUIP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QUIP_OK = 0,
  QUIP_ERR_ARG = 1,          /* null pointer, bad enum, bad bit width, ...   */
  QUIP_ERR_SHAPE = 2,        /* sizes inconsistent or unsupported            */
  QUIP_ERR_UNSUPPORTED = 3,  /* valid request this build does not implement  */
  QUIP_ERR_NOT_PD = 4,       /* LDL met a pivot <= 0 (H~ not positive definite) */
  QUIP_ERR_NONFINITE = 5,    /* NaN or Inf met on the device                 */
  QUIP_ERR_CUDA = 6,         /* a CUDA runtime / driver call failed          */
  QUIP_ERR_TIMEOUT = 7,      /* a bounded device-side wait ran out           */
  QUIP_ERR_WORKSPACE = 8     /* ws too small or misaligned                   */
} quip_status;

typedef enum { QUIP_F32 = 0, QUIP_BF16 = 1, QUIP_U8 = 2 } quip_dtype;

/* Kind of random orthogonal matrix on one side of W. */
typedef enum {
  QUIP_T_IDENTITY = 0,   /* no transform on this side                              */
  QUIP_T_HADAMARD = 1,   /* H_d diag(s) / sqrt(d), Sylvester order, s_i = +-1;
                            d a power of two, 2 <= d <= 8192                     */
  QUIP_T_KRONECKER = 2   /* A (x) B, A p x p, B q x q Haar-random, p * q = d,
                            1 <= p, q <= 256                                     */
} quip_tkind;

/* Flag OR'ed into a side's kind: a random permutation of the coordinates
 * before the structured factor T, S = T P with (P x)_r = x_{pi[r]} (QuIP,
 * Experiments, "Further Ablation" / Table 5: the random permutation step
 * within the fast orthogonal multiplication).  d <= 65536. */
#define QUIP_T_PERMUTE 0x100

/* Operations whose workspace quip_workspace_size() reports. */
typedef enum {
  QUIP_OP_INCOHERENCE_FORWARD = 0,
  QUIP_OP_INCOHERENCE_INVERSE = 1,
  QUIP_OP_LDL = 2,
  QUIP_OP_LDLQ = 3,
  QUIP_OP_GREEDY = 4,
  QUIP_OP_QMATVEC = 5
} quip_op;

typedef struct quip_transform quip_transform;   /* opaque, library-owned */

/* Human-readable name of a status code (static string, never NULL). */
const char* quip_status_string(int status);

/* Library version string, e.g. "quip-b200 0.1.0 sm_100a". */
const char* quip_version(void);

/* Number of CUDA kernels this library has enqueued since it was loaded
 * (all entry points, all streams; host-side counter). */
uint64_t quip_kernel_launches(void);

/*
 * Draw the two random orthogonal matrices for an m x n layer from `seed`
 * (QuIP, incoherence-processing section: U in O(m), V in O(n); QuIP# abstract:
 * randomized Hadamard).  Randomness: counter-based SplitMix64 (Steele, Lea &
 * Flood 2014); element i of stream t is output t*2^40 + i + 1 of the
 * sequence started at `seed`.  Streams: 0 = m-side signs, 1 = n-side signs,
 * 2 / 3 = m-side A / B Gaussians, 4 / 5 = n-side A / B Gaussians, 6 / 7 =
 * m-side / n-side permutation draws (pi lists the indices of the side's
 * first d draws in increasing order of the draw).  A sign is
 * -1 when the draw's top bit is set.  A Gaussian matrix element e (row-major)
 * is sqrt(-2 ln u1) cos(2 pi u2) with u = ((draw >> 11) + 1) 2^-53 of draws
 * 2e and 2e+1; the factor is Q of G = QR with diag(R) > 0.
 * Signs, factors and the QR are computed on the device on `stream`.
 *   m_kind / n_kind : quip_tkind for each side, optionally | QUIP_T_PERMUTE;
 *                     m_p*m_q == m for KRONECKER.
 *   out             : receives the new object (host pointer to a handle).
 * Allocates device memory owned by the object (freed by destroy).  The
 * object may be used on any stream after the creating stream has passed it.
 */
quip_status quip_transform_create(uint64_t seed, int64_t m, int64_t n,
                                  int m_kind, int64_t m_p, int64_t m_q,
                                  int n_kind, int64_t n_p, int64_t n_q,
                                  void* stream, quip_transform** out);

/*
 * Redraw an existing transform's random signs / factors from `seed` in place
 * (same definition as quip_transform_create, no allocation): kernels only,
 * enqueued on `stream`.  Work already enqueued that reads the transform must
 * be ordered before this call by the caller.
 */
quip_status quip_transform_draw(quip_transform* tf, uint64_t seed, void* stream);

/* Free a transform (synchronises the device first).  NULL is accepted. */
quip_status quip_transform_destroy(quip_transform* tf);

/*
 * Device pointers (library-owned, read-only, fp32) of one side's data:
 * side 0 = m side (U), 1 = n side (V).  For HADAMARD `signs` has d entries;
 * for KRONECKER `A` is p x p and `B` is q x q, row-major; pointers that do
 * not apply are set to NULL.  kind, p, q may be NULL.
 */
quip_status quip_transform_info(const quip_transform* tf, int side, int* kind,
                                int64_t* p, int64_t* q, const float** signs,
                                const float** A, const float** B);

/*
 * Device pointer (library-owned, read-only) of one side's permutation pi
 * (d int32, (P x)_r = x_{pi[r]}), or NULL when the side has none
 * (QUIP_T_PERMUTE not given).  side 0 = m side, 1 = n side.
 */
quip_status quip_transform_permutation(const quip_transform* tf, int side, const int32_t** perm);

/*
 * Proxy Hessian accumulation (QuIP, adaptive-rounding section: H is the
 * second moment of the calibration inputs): H_acc (+)= X^T X.
 *   X          : device, N x n, row stride ldx elements, dtype QUIP_BF16 or
 *                QUIP_F32.  For BF16 the bf16 products are exact and summed
 *                in fp32 on the tensor cores (tcgen05); ldx*2 must be a
 *                multiple of 16 bytes and X 16-byte aligned.
 *   H_acc      : device, n x n fp32, row stride n.  On return its lower
 *                triangle (i >= j) holds the (accumulated) sum; the strict
 *                upper triangle is unspecified until quip_hessian_finalize.
 *   accumulate : 0 = overwrite, 1 = add to the lower triangle already there
 *                (stream X in token chunks; N may differ per call).
 * N == 0 with accumulate == 0 writes zeros.  Token shards add: GPUs that each
 * accumulate their own tokens and sum H_acc (one all-reduce) before
 * quip_hessian_finalize with the total token count all hold the Hessian of
 * every token.
 */
quip_status quip_hessian_accumulate(const void* X, int dtype, int64_t N, int64_t n,
                                    int64_t ldx, float* H_acc, int accumulate,
                                    void* stream);

/*
 * H = sym(H_acc) / N_total + damp * mean(diag(H_acc / N_total)) * I, in place
 * (QuIP, Experiments, "Methods.": H <- H + alpha mean(diag H) I).  Reads the
 * lower triangle, writes the full symmetric matrix.  N_total >= 1, damp >= 0.
 */
quip_status quip_hessian_finalize(float* H, int64_t n, int64_t N_total, float damp,
                                  void* stream);

/*
 * Incoherence pre-processing (QuIP, incoherence-processing section):
 *   W_t = U W V^T   (m x n fp32, row stride n), W: device m x n, row stride
 *                   ldw, dtype QUIP_BF16 or QUIP_F32; W and W_t must not overlap;
 *                   skipped when W is NULL (then W_t, w_dtype and ldw are ignored);
 *   H   = V H V^T   in place (n x n fp32, full symmetric on entry and exit),
 *                   skipped when H is NULL.  W and H may not both be NULL.
 * The two are independent: a caller may transform H first (the LDL needs
 * only H~) and W later, e.g. while W is still being copied to the device.
 * When V is a Hadamard side with n >= 16, W (with ldw * element size a
 * multiple of 16 bytes), W_t and H must be 16-byte aligned (the row kernels
 * move 16-byte vectors), else QUIP_ERR_ARG.
 * ws: workspace for QUIP_OP_INCOHERENCE_FORWARD.
 */
quip_status quip_incoherence_forward(const quip_transform* tf, const void* W, int w_dtype,
                                     int64_t ldw, float* W_t, float* H, void* ws,
                                     size_t ws_bytes, void* stream);

/*
 * Incoherence post-processing: W_hat = U^T W_hat_t V (m x n fp32, row stride
 * n).  W_hat may equal W_hat_t (in place).  When V is a Hadamard side with
 * n >= 16 both must be 16-byte aligned, else QUIP_ERR_ARG.
 * ws: QUIP_OP_INCOHERENCE_INVERSE.
 */
quip_status quip_incoherence_inverse(const quip_transform* tf, const float* W_hat_t,
                                     float* W_hat, void* ws, size_t ws_bytes, void* stream);

/*
 * LDL factorisation H_t = (I + Ů) diag(D) (I + Ů)^T with Ů strictly upper
 * triangular (the factorisation that defines LDLQ's feedback; QuIP,
 * adaptive-rounding section).  In place on H_t (n x n fp32, row stride n,
 * symmetric positive definite; only the upper triangle is read; n % 4 == 0
 * and H_t 16-byte aligned):
 * on return the strict upper triangle holds Ů, D (device, n fp32) the
 * pivots; the diagonal and lower triangle of H_t are unspecified.
 * A pivot <= 0 or non-finite sets QUIP_ERR_NOT_PD in the status word
 * (quip_sync_status).  ws: QUIP_OP_LDL.
 * Part of the trailing update runs on a second stream of the current device
 * (created on first use, kept for the process); it forks from and joins back
 * into `stream` by events, so the call is ordered on `stream` like any other.
 */
quip_status quip_ldl(float* H_t, float* D, int64_t n, void* ws, size_t ws_bytes,
                     void* stream);

/*
 * LDLQ adaptive rounding of the incoherent weights (QuIP, adaptive-rounding
 * section; "Methods.": LDLQ = OPTQ), one b-bit per-row min/max grid:
 *   lo_i = min_j W_t[i,j], s_i = (max_j W_t[i,j] - lo_i) / (2^bits - 1)
 *   (s_i = 1 for a constant row);
 *   for k = 0..n-1: a_k = W_t[:,k] + sum_{j<k} (W_t[:,j] - W^[:,j]) Ů[j,k],
 *   codes[:,k] = clamp(rint((a_k - lo) / s), 0, 2^bits - 1) (ties to even),
 *   W^[:,k] = lo + s codes[:,k].
 * Evaluated in fp32, blocked over `block` columns (the result does not
 * depend on block in exact arithmetic).
 *   W_t   : device m x n fp32 (row stride n), not modified.
 *   Uring : device n x n fp32, row stride ldu >= n (ldu % 4 == 0); only the
 *           strict upper triangle is read (the H_t buffer quip_ldl returned).
 *           W_t and Uring 16-byte aligned.
 *   bits  : 1..8.  block: 32, 64 or 128, with n % block == 0 and n % 64 == 0;
 *           a performance hint only (the result does not depend on it in
 *           exact arithmetic): this build always processes 128-column
 *           blocks (the last one 64 wide when n % 128 == 64).
 *   codes : device m x n uint8 (row stride n).  lo, scale: device m fp32.
 * ws: QUIP_OP_LDLQ.
 */
quip_status quip_ldlq_quantize(const float* W_t, const float* Uring, int64_t ldu,
                               int64_t m, int64_t n, int bits, int64_t block,
                               uint8_t* codes, float* lo, float* scale, void* ws,
                               size_t ws_bytes, void* stream);

/*
 * Size of the device array quip_ldlq_quantize_static uses as its workspace.
 */
#define QUIP_LDLQ_STATIC_SCRATCH_BYTES (16u << 20)

/*
 * quip_ldlq_quantize without a caller-supplied workspace and without any
 * device allocation.  This entry point has no counterpart in the QuIP papers;
 * it exists for callers that cannot call cudaMalloc: programs whose device
 * memory is owned by a fixed pool or arena handed out by their own runtime,
 * programs running under a hard memory cap, and latency-sensitive callers
 * that must not trigger the device-wide synchronisation that cudaMalloc and
 * cudaFree can cause.
 *
 * Same arguments, results and errors as quip_ldlq_quantize, minus (ws,
 * ws_bytes).  The workspace is a fixed array of QUIP_LDLQ_STATIC_SCRATCH_BYTES
 * in the library's own device memory, present on every GPU that loads the
 * library until the process exits.  Layers whose workspace
 * (quip_workspace_size(QUIP_OP_LDLQ, ...)) is larger are rejected with
 * QUIP_ERR_WORKSPACE before anything is launched.
 *  - Every call outside stream capture looks up the array's device address
 *    on the current device (so a cudaDeviceReset in between is harmless); a
 *    call whose stream is capturing reuses the address of the last call
 *    outside capture on that device, so make one call on each device before
 *    capturing (a device never called outside capture returns
 *    QUIP_ERR_CUDA), and none between a cudaDeviceReset and a capture.
 *  - Every call on a device shares the one array and it keeps the last
 *    call's contents; nothing in it needs to start at zero (every call
 *    overwrites what it reads).  Calls whose work overlaps on the GPU
 *    (different streams, or host threads) race on the array: order them.
 */
quip_status quip_ldlq_quantize_static(const float* W_t, const float* Uring, int64_t ldu,
                                      int64_t m, int64_t n, int bits, int64_t block,
                                      uint8_t* codes, float* lo, float* scale, void* stream);

/*
 * Nearest rounding (QuIP, Experiments, "Methods.": the nearest-rounding
 * baseline) on the per-row grid of quip_ldlq_quantize:
 *   lo, scale as there; codes[i,j] = clamp(rint((W_t[i,j] - lo_i) / s_i), 0, 2^bits - 1)
 * with the same fp32 steps as LDLQ's rounding (the quotient is formed as
 * (W_t - lo) * (1 / s)).  W_t: device m x n fp32, row stride n; codes:
 * device m x n uint8; lo, scale: device m fp32.  bits 1..8.
 */
quip_status quip_nearest_quantize(const float* W_t, int64_t m, int64_t n, int bits,
                                  uint8_t* codes, float* lo, float* scale, void* stream);

/*
 * LDLQ-RG's quantisation order (QuIP, Experiments, "Methods.": LDLQ-RG
 * re-orders the weights by diag(H)): perm[r] = the index k with the r-th
 * largest H[k,k] (equal values by increasing k; -0 counts as +0; where a
 * NaN goes is unspecified), iperm[perm[r]] = r.
 *   H     : device, n x n fp32, row stride ldh; only the diagonal is read.
 *   perm  : device n int32;  iperm: device n int32, or NULL.
 * n <= 65536.
 */
quip_status quip_diag_order(const float* H, int64_t ldh, int64_t n, int32_t* perm, int32_t* iperm,
                            void* stream);

/*
 * Gather out[r,c] = in[row_perm[r], col_perm[c]] (device; rows x cols,
 * row strides ldin / ldout elements; a NULL list is the identity), for
 * dtype QUIP_F32, QUIP_BF16 or QUIP_U8 (in and out of the same type, bits
 * copied unchanged).  With perm from quip_diag_order, col_perm = perm puts
 * a matrix's columns in the quantisation order and col_perm = iperm puts
 * them back.  in and out must not overlap.  An index outside
 * [0, rows) / [0, cols) writes 0 there and sets QUIP_ERR_ARG in the status
 * word (quip_sync_status).
 */
quip_status quip_permute(const void* in, int dtype, int64_t rows, int64_t cols, int64_t ldin,
                         const int32_t* row_perm, const int32_t* col_perm, void* out, int64_t ldout,
                         void* stream);

/*
 * Greedy updates of the proxy tr((W^ - W_t) H (W^ - W_t)^T) (QuIP,
 * Experiments, "Methods.": "Greedy" performs them alone, LDLQ-RG after
 * LDLQ), `passes` passes.  A pass visits k = 0..n-1 and, every other column
 * held at its current value, sets
 *   codes[:,k] = clamp(rint((t_k - lo) / s), 0, 2^bits - 1),
 *   t_k = W_t[:,k] - sum_{j != k} (W^[:,j] - W_t[:,j]) H[j,k] / H[k,k],
 * W^ = lo + s codes: per row, the grid point that minimises the proxy over
 * column k.  Evaluated in fp32 (tensor-core GEMMs on three bf16 pieces for
 * the long sums, as LDLQ's); the grid (lo, scale) is not changed.
 *   W_t   : device m x n fp32 (row stride n, 16-byte aligned), not modified.
 *   H     : device n x n fp32, symmetric with a positive diagonal, row stride
 *           ldh >= n; only the upper triangle (j <= k) is read.
 *   lo, scale : device m fp32 (e.g. from quip_ldlq_quantize).
 *   codes : device m x n uint8 (row stride n, 16-byte aligned), in: the
 *           starting codes, out: the codes after the passes.
 * n % 64 == 0, n <= 65536, m <= 2^20, bits 1..8, passes >= 0 (0: nothing
 * is done).  To visit the columns in another order, permute W_t's columns
 * and H's rows and columns first (quip_permute).  ws: QUIP_OP_GREEDY.
 */
quip_status quip_greedy_refine(const float* W_t, const float* H, int64_t ldh, int64_t m, int64_t n,
                               int bits, const float* lo, const float* scale, uint8_t* codes,
                               int passes, void* ws, size_t ws_bytes, void* stream);

/*
 * 32-bit words per row of packed codes (the smallest valid ldp of
 * quip_pack_codes / quip_qmatvec): ceil(n / (32 / slot)) rounded up to a
 * multiple of 4, slot = bits for bits in {1, 2, 4, 8}, 4 for bits 3, 8 for
 * bits 5..7.  Host only; 0 for invalid arguments.
 */
int64_t quip_packed_words(int64_t n, int bits);

/*
 * Pack b-bit codes for the quantized product (the pages print no storage
 * format; this is the library's): code j of row i goes to word
 * j mod Wd of row i at bit (j div Wd) * slot, Wd = quip_packed_words(n,
 * bits); unused slots are 0.
 *   codes  : device m x n uint8 (row stride n), values < 2^bits (higher
 *            bits are dropped).
 *   packed : device m x ldp uint32, ldp >= Wd, ldp % 4 == 0, 16-byte aligned.
 */
quip_status quip_pack_codes(const uint8_t* codes, int64_t m, int64_t n, int bits, uint32_t* packed,
                            int64_t ldp, void* stream);

/*
 * The quantized layer times B full-precision vectors (QuIP, Experiments,
 * "Throughput Comparison.": quantized matrix times full-precision vector,
 * with the incoherence processing around it):
 *   y_b = U^T (lo + s codes) V x_b     for b < B  (W^ = U^T W~^ V, the layer
 *   the pipeline's inverse transform returns),
 * computed as x' = V x (the transform's row kernels), z_i = lo_i sum(x') +
 * s_i sum_j c_ij x'_j (one kernel over the packed codes, fp32 sums), y = U^T z.
 *   tf     : the layer's transform (m x n).
 *   packed : from quip_pack_codes with the same bits; row stride ldp words.
 *   lo, scale : device m fp32 (the grid of the codes).
 *   x      : device B x n, row stride ldx elements, QUIP_F32 or QUIP_BF16
 *            (16-byte aligned rows when V is a Hadamard side without
 *            permutation and n >= 16).
 *   y      : device B x m fp32, row stride ldy.
 * n % 4 == 0.  The product kernel takes the vectors 8 at a time (4 for
 * 1-bit codes).  ws: QUIP_OP_QMATVEC with block = B.
 */
quip_status quip_qmatvec(const quip_transform* tf, const uint32_t* packed, int64_t ldp, const float* lo,
                         const float* scale, int bits, const void* x, int x_dtype, int64_t ldx, int64_t B,
                         float* y, int64_t ldy, void* ws, size_t ws_bytes, void* stream);

/* W_hat_t[i,j] = lo[i] + scale[i] * codes[i,j]  (device; m x n, row stride n). */
quip_status quip_dequantize(const uint8_t* codes, const float* lo, const float* scale,
                            int64_t m, int64_t n, float* W_hat_t, void* stream);

/*
 * Bytes of workspace `op` needs (quip_op).  tf is required for the
 * incoherence ops and QUIP_OP_QMATVEC and ignored otherwise; block is used
 * by QUIP_OP_LDLQ, and is the number of vectors B for QUIP_OP_QMATVEC
 * (whose m and n come from tf); QUIP_OP_GREEDY takes m and n.
 * *bytes may be 0.
 */
quip_status quip_workspace_size(int op, const quip_transform* tf, int64_t m, int64_t n,
                                 int64_t block, size_t* bytes);

/*
 * The whole path for one layer, from the problem statement of the QuIP page
 * (W, calibration inputs X, bit width, damping, LDLQ block size, seed):
 * draw (U, V) from `seed` into tf (quip_transform_draw), H = X^T X / N
 * (quip_hessian_accumulate), damping (quip_hessian_finalize, alpha = damp),
 * H~ = V H V^T and the LDL of H~ (quip_incoherence_forward, quip_ldl),
 * W~ = U W V^T and LDLQ (quip_ldlq_quantize), then, when W_hat is not NULL,
 * W^ = U^T (lo + s codes) V (quip_dequantize, quip_incoherence_inverse);
 * each step has the arguments, layout and errors of its own entry point.
 * The Hessian path (V, H, H~, the LDL) runs on a library-owned stream of the
 * highest priority, forked from and joined into `stream`; the weight path
 * (U, W~, LDLQ's per-row grid and the start of its accumulator) runs on
 * `stream` beside it; the rest of LDLQ and W^ follow on `stream`.  The codes and grid are those of LDLQ in the
 * incoherent basis (quip_ldlq_quantize); W^ is the dequantised layer in the
 * original basis.
 *   tf       : a transform made for this layer's m x n (quip_transform_create);
 *              it is redrawn from `seed`.
 *   W        : device, m x n, w_dtype QUIP_F32 or QUIP_BF16, row stride ldw.
 *   X        : device, N x n (N >= 1 tokens), x_dtype QUIP_F32 or QUIP_BF16,
 *              row stride ldx.
 *   bits     : 1 .. 8.  block: 32, 64 or 128 with n % block == 0 and n % 64 == 0;
 *              a performance hint, as for quip_ldlq_quantize.
 *   damp     : alpha >= 0.
 *   codes    : device m x n uint8.  lo, scale: device m fp32.
 *   W_hat    : device m x n fp32, or NULL to stop after the codes.
 * ws: quip_layer_workspace_size(tf, N, w_dtype, x_dtype, block, 0, ...).
 * On return ws holds, at offset 0, the n x n fp32 matrix whose strict upper
 * triangle is Ů (as quip_ldl leaves it); at a = round256(4 n^2) the n pivots
 * D (fp32); at a + round256(4 n) W~ (m x n fp32); round256(x) rounds x up to
 * a multiple of 256.
 * Device-side errors (non-PD H~, non-finite values) go to the status word.
 */
quip_status quip_quantize_layer(quip_transform* tf, uint64_t seed, const void* W, int w_dtype,
                                int64_t ldw, const void* X, int x_dtype, int64_t N, int64_t ldx,
                                int bits, int64_t block, float damp, uint8_t* codes, float* lo,
                                float* scale, float* W_hat, void* ws, size_t ws_bytes, void* stream);

/*
 * quip_quantize_layer from host memory to host memory.  W_host, X_host
 * (same shapes, types and strides as above) are copied to the device on a
 * library-owned copy stream, X in token chunks of at least 2048 so that the
 * Hessian accumulates each chunk as it lands, W while the Hessian, H~ and the
 * LDL run (they do not read W); codes_host (m x n uint8) is copied back on
 * that stream in column chunks (about eight, one cudaMemcpy2DAsync each) as
 * LDLQ finishes their columns, lo_host and scale_host (m fp32) once LDLQ is
 * done, and W^ (m x n fp32) into W_hat_host when it is not NULL (W^ is
 * computed either way: it is the last step of the path).  One
 * cudaMemcpy2DAsync / cudaMemcpyAsync per piece.  `stream` waits for every
 * copy, so synchronising it makes all host outputs valid; host buffers
 * should be page-locked for the copies to overlap the kernels.  All device
 * buffers live in ws: quip_layer_workspace_size(tf, N, w_dtype, x_dtype,
 * block, 1, ...).
 */
quip_status quip_quantize_layer_host(quip_transform* tf, uint64_t seed, const void* W_host,
                                     int w_dtype, int64_t ldw, const void* X_host, int x_dtype,
                                     int64_t N, int64_t ldx, int bits, int64_t block, float damp,
                                     uint8_t* codes_host, float* lo_host, float* scale_host,
                                     float* W_hat_host, void* ws, size_t ws_bytes, void* stream);

/*
 * Device workspace of quip_quantize_layer (host = 0) or
 * quip_quantize_layer_host (host = 1) for N tokens and the given types:
 * H~ (n x n fp32), D, W~ (m x n fp32), the largest stage workspace and the
 * weight path's own region (its transform's workspace, then LDLQ's m x n
 * fp32 accumulator); the host variant adds device copies of W and X, the
 * codes, the grid and W^.
 */
quip_status quip_layer_workspace_size(const quip_transform* tf, int64_t N, int w_dtype, int x_dtype,
                                      int64_t block, int host, size_t* bytes);

/*
 * Per-kernel device timing, for measurement (the QuIP papers have no
 * counterpart).  quip_timing_begin() discards earlier records and turns
 * timing on: from then on every kernel the library launches, on any stream,
 * is bracketed by two CUDA events recorded on its own stream and filed under
 * the kernel's name.  quip_timing_end() turns timing off, waits for the
 * recorded events, and writes up to max_entries aggregates, largest total
 * first: names[i] (static string owned by the library), launches[i] and
 * total_ms[i] (sum of the launches' event-measured durations).
 * *n_entries receives the number of distinct kernels recorded.  The events
 * add a few microseconds of host work per launch; time a run without them
 * for throughput.  Not meant for concurrent use from several host threads.
 */
quip_status quip_timing_begin(void);
quip_status quip_timing_end(const char** names, uint64_t* launches, double* total_ms,
                            int max_entries, int* n_entries);

/*
 * The launches recorded since quip_timing_begin() one by one, in the order
 * they were enqueued (instead of quip_timing_end's aggregates; either call
 * ends the recording and discards the records): names[i], start_ms[i] and
 * end_ms[i] (the launch's two events, in ms after the first launch's start
 * event) and stream_ids[i] (streams numbered in order of first appearance),
 * for i < min(max_entries, *n_entries); *n_entries receives the number of
 * launches recorded.  A timeline of the streams' overlap; the events between
 * launches break programmatic dependent launch, so the gaps are upper bounds.
 */
quip_status quip_timing_trace(const char** names, double* start_ms, double* end_ms, int* stream_ids,
                              int max_entries, int* n_entries);

/*
 * Synchronise `stream`, then return and clear the device status word
 * (QUIP_OK if no device-side error was recorded since the last call), or
 * QUIP_ERR_CUDA if a CUDA error is pending.  The status word is shared by all
 * streams of the process on the current device.
 */
quip_status quip_sync_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QUIP_H_ */
