/*
 * tq.h -- C ABI of the B200 (sm_100a) W4A4 + low-rank linear layer.
 *
 *   Y = dequant( Q4(X H) . Q4(H^T R) ) + (X L1) L2
 *
 * H is the block-diagonal Sylvester Hadamard matrix (block b along K,
 * normalised by 1/sqrt(b)); Q4 is the symmetric 4-bit quantizer of CoQuant
 * Eq. (1) (zero-point 0, s = max|.| / 7, RoundClip to [-7, 7]), applied per
 * token to the rotated activations and per output channel to the rotated
 * residual; the integer product accumulates in INT32 (TwinQuant notes,
 * section 04.C, Figure 4); the bf16 low-rank branch (X L1) L2 is the U V term
 * of the SVDQuant-style split (TwinQuant notes, section 02.A) and both
 * branches meet in one epilogue (TwinQuant, "single epilogue" of the fused
 * dual-component kernel).  The rotation rests on CoQuant Eq. (3):
 * (X H)(H^T W) = X W for orthogonal H.
 *
 * Conventions shared by every entry point:
 *  - All array pointers are DEVICE pointers owned by the caller; the library
 *    allocates nothing on these paths.  Calls are asynchronous on `stream`
 *    (a cudaStream_t passed as void*, NULL = legacy default stream).
 *  - Matrices are row-major with K (the reduction / in-feature dimension)
 *    contiguous, the nn.Linear [out][in] convention: X [M][K], R^T [N][K],
 *    L1^T [r][K], L2^T [N][r], Y [M][N].  bf16 data is passed as uint16_t
 *    bit patterns.
 *  - Packed int4 codes ("Xq", "Wq") are [rows][K/2] bytes.  Within every
 *    group of 32 consecutive codes (16 bytes) byte i holds code i in the low
 *    nibble and code i+16 in the high nibble, each a 4-bit two's complement
 *    number in [-7, 7] (-8 is never produced).
 *  - Scales are fp32: s_x[m] = max_k |(X H)[m,k]| / 7, s_w[n] likewise over
 *    row n of R^T H.  A row that is all zero gets scale 0 and all codes 0.
 *  - Shape limits: M >= 1; 128 <= K <= 32768 with K % 128 == 0;
 *    had_block in {1, 2, 4, ..., 256} (1 = no rotation) dividing K;
 *    N >= 8 with N % 8 == 0; r = 0 or a multiple of 16 up to 512.
 *    Every pointer must be 16-byte aligned.
 *  - Inputs must be finite.  Rounding is round-half-to-even everywhere.
 *  - Errors are returned synchronously before anything is launched
 *    (TQ_ERR_INVALID_VALUE, TQ_ERR_UNSUPPORTED_SHAPE, TQ_ERR_MISALIGNED,
 *    TQ_ERR_WORKSPACE, TQ_ERR_NO_DEVICE); a failed launch returns
 *    TQ_ERR_CUDA.  Kernel-side watchdog timeouts (a pipeline wait that never
 *    completes) are recorded in the GEMM workspace and reported by
 *    tq_query_device_status.  No call aborts the process.
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TQ_API __attribute__((visibility("default")))
#else
#define TQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TQ_OK = 0,
  TQ_ERR_INVALID_VALUE = 1,     /* null pointer, non-positive size          */
  TQ_ERR_UNSUPPORTED_SHAPE = 2, /* shape outside the limits above           */
  TQ_ERR_MISALIGNED = 3,        /* a pointer is not 16-byte aligned         */
  TQ_ERR_CUDA = 4,              /* CUDA launch or runtime error             */
  TQ_ERR_TIMEOUT = 5,           /* a kernel's bounded wait gave up          */
  TQ_ERR_WORKSPACE = 6,         /* workspace missing or too small           */
  TQ_ERR_NO_DEVICE = 7          /* current device is not an sm_100 GPU      */
} tq_status;

/* Human-readable name of a status code (static string, never NULL). */
TQ_API const char* tq_status_string(int status);

/* ABI version of this library (major * 100 + minor). */
TQ_API int tq_version(void);

/*
 * tq_pack_weight -- offline rotation + per-output-channel INT4 quantization
 * of the residual (CoQuant Eq. (3): the weight side of (X H)(H^T W); Eq. (1)
 * per channel; CoQuant's protocol uses per-channel symmetric weights).
 *
 *   Rt   [N][K] fp32  in : R^T, the residual in nn.Linear layout
 *   Wq   [N][K/2] u8 out : packed int4 codes of row n of R^T H
 *   s_w  [N] fp32    out : per-channel scales
 * Not on the per-token path: run once per layer.
 */
TQ_API int tq_pack_weight(const float* Rt, int N, int K, int had_block,
                   uint8_t* Wq, float* s_w, void* stream);

/*
 * tq_quantize_act -- online rotation X H (CoQuant Eq. (3), block Hadamard),
 * symmetric per-token INT4 quantization (CoQuant Eq. (1); TwinQuant notes
 * section 02) and the low-rank down-projection X L1 (TwinQuant notes
 * section 02.A).  Two kernels serve it:
 *  - M >= 64 with had_block <= 128: 128-token tiles on the tensor cores.  The
 *    rotation of each 128-column block is a bf16 MMA against the
 *    block-diagonal +-1 Sylvester matrix (exact products, fp32 accumulation)
 *    and X L1 a second MMA on the same staged tile.  X is read twice: the
 *    first pass takes the per-token absmax across a thread-block cluster,
 *    the second (served from L2) recomputes the rotation and writes codes.
 *    Ranks above 128 run X L1 in extra launches of at most 256 columns.
 *  - otherwise (few tokens, or had_block = 256): an in-register and
 *    warp-shuffle fast Walsh-Hadamard transform per block, X L1 on mma.sync,
 *    all from one read of X; K is split over a thread-block cluster that
 *    combines the absmax and the X L1 partials in distributed shared memory.
 * Both give the same codes up to the midpoint allowance of the fp32
 * summation order.
 *
 *   X    [M][K] bf16    in : activations
 *   L1t  [r][K] bf16    in : L1^T (down-projection weight); NULL iff r == 0
 *   Xq   [M][K/2] u8   out : packed codes of X H
 *   s_x  [M] fp32      out : per-token scales
 *   XL1  [M][r] fp32   out : X L1 (unrotated, unquantized X); NULL iff r == 0
 */
TQ_API int tq_quantize_act(const uint16_t* X, int M, int K, int had_block,
                    const uint16_t* L1t, int r,
                    uint8_t* Xq, float* s_x, float* XL1, void* stream);

/*
 * Bytes of device workspace tq_w4a4_lr_gemm needs for this shape (always at
 * least 256).  The workspace must be zero-filled once before its first use;
 * every call leaves its counters zero again, so it can be reused by later
 * calls on the same stream (not by concurrent calls).
 */
TQ_API size_t tq_gemm_workspace_bytes(int M, int N, int K, int r);

/*
 * tq_w4a4_lr_gemm -- the layer's main kernel (TwinQuant's fused
 * dual-component kernel, bf16 low-rank form):
 *
 *   Y[m][n] = bf16( s_x[m] s_w[n] sum_k qx[m][k] qw[n][k]
 *                   + sum_j bf16(XL1[m][j]) L2t[n][j] )
 *
 * the integer sum exact in INT32, the low-rank sum in fp32.
 *   Xq, s_x, XL1   : outputs of tq_quantize_act (XL1 NULL iff r == 0)
 *   Wq, s_w        : outputs of tq_pack_weight
 *   L2t [N][r] bf16: L2^T (up-projection weight); NULL iff r == 0
 *   Y   [M][N] bf16: output
 *   workspace      : >= tq_gemm_workspace_bytes(M, N, K, r) bytes, zeroed
 *                    before first use (see above)
 */
TQ_API int tq_w4a4_lr_gemm(const uint8_t* Xq, const float* s_x,
                    const uint8_t* Wq, const float* s_w,
                    const float* XL1, const uint16_t* L2t,
                    int M, int N, int K, int r, uint16_t* Y,
                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * tq_w4a4_lr_layer -- the whole layer from bf16 activations:
 *
 *   Y = bf16( s_x s_w (Q4(X H) . Wq) + bf16(X L1) L2 )
 *
 * i.e. tq_quantize_act followed by tq_w4a4_lr_gemm, with the same codes,
 * scales and tolerances.  At decode sizes (M <= 16, r in {0, 16, 32, 64},
 * K % 256 == 0, K <= 4096, K / 256 dividing 16 at rank 64, had_block <=
 * 256) it runs as ONE kernel
 * (TwinQuant notes section 04.C: the residual GEMM quantizes activations
 * concurrently and both paths share one epilogue): a thread-block cluster
 * of K / 256 CTAs per group of output channels, each CTA rotating its
 * 256-column slice of X with the same butterflies as tq_quantize_act (so
 * the codes and scales are the same), exchanging the per-token absmax, the
 * X L1 partials and the split-K sums in distributed shared memory, and
 * feeding the codes to tcgen05 integer MMAs whose int4 weights were
 * requested and expanded into tensor memory before the kernel waited on
 * its predecessor.  Two such CTAs (two consecutive layers) share an SM.
 * For M > 128 with had_block <= 128 it runs
 * tq_quantize_act_i8 + tq_w4a4_lr_gemm_a8 (codes one per byte in the
 * workspace).  Other shapes run tq_quantize_act + tq_w4a4_lr_gemm, keeping
 * Xq, s_x and XL1 in the workspace.
 *
 *   X [M][K] bf16, L1t [r][K] bf16 (NULL iff r == 0), Wq [N][K/2] u8,
 *   s_w [N] fp32, L2t [N][r] bf16 (NULL iff r == 0), Y [M][N] bf16 (out)
 *   The weights (Wq, s_w, L1t, L2t) may be read before the kernel waits for
 *   the work queued before it on `stream` (programmatic dependent launch):
 *   they must not be written by the kernel launched immediately before
 *   this call on the same stream, unless that kernel makes its stores
 *   visible before it exits (the library's pack kernels do).
 *   workspace: >= tq_layer_workspace_bytes(M, N, K, r) bytes, zero-filled
 *   before first use (its first 4 bytes are the watchdog status word)
 */
TQ_API size_t tq_layer_workspace_bytes(int M, int N, int K, int r);
TQ_API int tq_w4a4_lr_layer(const uint16_t* X, const uint16_t* L1t,
                            const uint8_t* Wq, const float* s_w,
                            const uint16_t* L2t, int M, int N, int K, int r,
                            int had_block, uint16_t* Y,
                            void* workspace, size_t workspace_bytes,
                            void* stream);

/*
 * tq_layer_path -- which kernels tq_w4a4_lr_layer runs for a shape.  A host
 * query: no device work, no CUDA call.  Returns TQ_PATH_FUSED (the one-kernel
 * decode layer), TQ_PATH_CODES_I8 (tq_quantize_act_i8 + tq_w4a4_lr_gemm_a8),
 * TQ_PATH_CODES_PACKED (tq_quantize_act + tq_w4a4_lr_gemm), or the negative
 * of the tq_status tq_w4a4_lr_layer would return for the shape's arguments
 * (TQ_ERR_INVALID_VALUE, TQ_ERR_UNSUPPORTED_SHAPE).
 */
enum { TQ_PATH_FUSED = 0, TQ_PATH_CODES_I8 = 1, TQ_PATH_CODES_PACKED = 2 };
TQ_API int tq_layer_path(int M, int N, int K, int r, int had_block);

/*
 * Shared input, gate / up pair with a SwiGLU epilogue (the MLP's gate and
 * up projections read the same X, so its rotation, codes and X L1 are
 * computed once for both; TwinQuant notes section 04.C: one shared epilogue).
 *
 * tq_pack_gate_up -- offline: the two projections' packed operands (each as
 * tq_pack_weight makes them, with rank r) as one layer of 2N channels:
 *   Wq2  [2N][K/2] u8   row 2i = gate row i, row 2i+1 = up row i
 *   s_w2 [2N] fp32      interleaved the same way
 *   L1t2 [2r][K] bf16   gate L1^T rows, then up L1^T rows
 *   L2t2 [2N][2r] bf16  row 2i = [gate L2^T row i, 0], row 2i+1 = [0, up row i]
 * L1t_* / L2t_* / L1t2 / L2t2 are NULL iff r == 0; 2r <= 512.
 *
 * tq_w4a4_lr_gate_up -- Y[t][i] = bf16( silu(g) * u ), silu(g) = g / (1 + e^-g),
 * with g and u the fp32 layer outputs (s_x s_w acc + lr, before any rounding)
 * of gate channel i and up channel i.  One activation pass (codes one per
 * byte, X L1 of rank r2 = 2r) and one int8-code GEMM over the 2N channels,
 * whose epilogue pairs the two rows of each channel.
 *   X [M][K] bf16, the pair from tq_pack_gate_up, Y [M][N] bf16 (out);
 *   workspace >= tq_gate_up_workspace_bytes(M, N, K, r2), zero-filled before
 *   first use.  Limits: had_block <= 128, N % 8 == 0, r2 % 32 == 0, r2 <= 512.
 */
TQ_API int tq_pack_gate_up(const uint8_t* Wq_g, const float* s_w_g, const uint16_t* L1t_g,
                           const uint16_t* L2t_g, const uint8_t* Wq_u, const float* s_w_u,
                           const uint16_t* L1t_u, const uint16_t* L2t_u, int N, int K, int r,
                           uint8_t* Wq2, float* s_w2, uint16_t* L1t2, uint16_t* L2t2,
                           void* stream);
TQ_API size_t tq_gate_up_workspace_bytes(int M, int N, int K, int r2);
TQ_API int tq_w4a4_lr_gate_up(const uint16_t* X, const uint16_t* L1t2, const uint8_t* Wq2,
                              const float* s_w2, const uint16_t* L2t2, int M, int N, int K,
                              int r2, int had_block, uint16_t* Y, void* workspace,
                              size_t workspace_bytes, void* stream);

/*
 * Shared input, any n <= 8 projections (Q, K and V of attention; CoQuant's
 * note that layers sharing an input share one transform, Eq. (14)): the
 * projections as ONE layer, so that one activation pass (rotation, codes,
 * X L1 of the stacked ranks) and one GEMM serve them all.
 *
 * tq_pack_shared_input -- offline, copies only: projection i's operands
 * (as tq_pack_weight makes them, rank r[i], N[i] channels; host arrays of n
 * device pointers, L1t[i] / L2t[i] NULL iff r[i] == 0) concatenated:
 *   Wq_cat  [sum N][K/2] u8   projection 0's rows, then 1's, ...
 *   s_w_cat [sum N] fp32      likewise
 *   L1t_cat [sum r][K] bf16   L1^T rows stacked along the rank
 *   L2t_cat [sum N][sum r]    block-diagonal: rows of projection i hold its
 *                             L2^T in columns [sum_{j<i} r[j], +r[i]), zeros
 *                             elsewhere (exact zeros: they add nothing)
 * L1t_cat and L2t_cat are NULL iff sum r == 0.  Limits: N[i] % 8 == 0,
 * r[i] % 16 == 0, sum r <= 512.  Asynchronous on `stream`.
 * Run the result through tq_w4a4_lr_layer (N = sum N, r = sum r): its Y
 * [M][sum N] holds projection i's Y in columns [sum_{j<i} N[j], +N[i]),
 * with the codes, integer sums and tolerances of that projection alone.
 */
TQ_API int tq_pack_shared_input(int n, const uint8_t* const* Wq, const float* const* s_w,
                                const uint16_t* const* L1t, const uint16_t* const* L2t,
                                const int* N, const int* r, int K, uint8_t* Wq_cat,
                                float* s_w_cat, uint16_t* L1t_cat, uint16_t* L2t_cat,
                                void* stream);

/*
 * Randomized Hadamard transform (the TORQUE page, randomized Hadamard
 * abstract: random signs, then the Hadamard): the rotation U of CoQuant
 * Eq. (3) becomes D H, with D = diag(d) a +-1 sign vector, on both sides:
 * activations x -> x D H, weights R -> (D H)^T R (row n of R^T D H).  D H is
 * orthogonal, so Eq. (3) still gives (x D H)((D H)^T W) = x W.  The signs are
 * a device bit mask of K / 32 uint32 words: bit (k % 32) of word k / 32 set
 * means d_k = -1.  X L1 reads the unrotated X and is unchanged.
 *
 * tq_pack_weight_rht   -- tq_pack_weight with D H.
 * tq_quantize_act_rht  -- tq_quantize_act with D H, on the same kernels:
 *                         the butterflies (sign flips in registers before
 *                         them), or for M >= 64 with had_block <= 128 the
 *                         tensor-core kernel, which negates the masked
 *                         columns of each staged X block (and of L1^T, so
 *                         X L1 is unchanged) in shared memory before its
 *                         MMAs.  Sign flips are exact either way.
 * tq_w4a4_lr_layer_rht -- tq_w4a4_lr_layer with D H (weights from
 *                         tq_pack_weight_rht with the same mask): the
 *                         one-kernel decode layer where it applies; for
 *                         M > 128 with had_block <= 128 the tensor-core
 *                         activation kernel writing one code per byte and
 *                         bf16(X L1), then tq_w4a4_lr_gemm_a8; else
 *                         tq_quantize_act_rht + tq_w4a4_lr_gemm (packed
 *                         codes).  tq_layer_path reports the same choice.
 * Arguments and limits as the plain calls; `signs` 16-byte aligned.
 */
TQ_API int tq_pack_weight_rht(const float* Rt, int N, int K, int had_block,
                              const uint32_t* signs, uint8_t* Wq, float* s_w, void* stream);
TQ_API int tq_quantize_act_rht(const uint16_t* X, int M, int K, int had_block,
                               const uint32_t* signs, const uint16_t* L1t, int r, uint8_t* Xq,
                               float* s_x, float* XL1, void* stream);
TQ_API int tq_w4a4_lr_layer_rht(const uint16_t* X, const uint32_t* signs, const uint16_t* L1t,
                                const uint8_t* Wq, const float* s_w, const uint16_t* L2t,
                                int M, int N, int K, int r, int had_block, uint16_t* Y,
                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * Composed randomized Hadamard transforms (two make every coordinate's
 * marginal near-Gaussian, three also decorrelate blocks of coordinates for
 * vector quantization): x D_1 H D_2 H ... D_n H
 * with n = n_rht in 1..3 masks, stored one after another in `signs`
 * ([n_rht][K / 32] words, the first applied first); weights packed by
 * tq_pack_weight_rhtn with the same masks.  The _rht calls above are
 * n_rht = 1.  For n_rht > 1 the activations take the butterfly kernel at
 * every M (above 128 tokens writing one code per byte for the int8-code
 * GEMM).  Same arguments and limits otherwise.
 */
TQ_API int tq_pack_weight_rhtn(const float* Rt, int N, int K, int had_block,
                               const uint32_t* signs, int n_rht, uint8_t* Wq, float* s_w,
                               void* stream);
TQ_API int tq_quantize_act_rhtn(const uint16_t* X, int M, int K, int had_block,
                                const uint32_t* signs, int n_rht, const uint16_t* L1t, int r,
                                uint8_t* Xq, float* s_x, float* XL1, void* stream);
TQ_API int tq_w4a4_lr_layer_rhtn(const uint16_t* X, const uint32_t* signs, int n_rht,
                                 const uint16_t* L1t, const uint8_t* Wq, const float* s_w,
                                 const uint16_t* L2t, int M, int N, int K, int r, int had_block,
                                 uint16_t* Y, void* workspace, size_t workspace_bytes,
                                 void* stream);

/*
 * Per-token asymmetric activations (CoQuant Eq. (1) with a zero-point; the
 * protocol CoQuant follows quantizes activations per token asymmetrically):
 * for each token's rotated row v, z = min(v), s = (max(v) - min(v)) / 15,
 * q = RoundClip((v - z) / s) in [0, 15] (ties to even), Q(v) = s q + z.  A
 * constant row gets s = 0 and codes 0.
 *
 * tq_quantize_act_asym_i8 -- as tq_quantize_act_i8, with Xq8 = q - 8 (int8
 * in [-8, 7]), s_x [M] = s and z_x [M] = z of the normalised rotation.
 * tq_weight_code_sums -- offline: wsum [N] int32 = sum_k of each channel's
 * weight codes (from Wq as tq_pack_weight makes it).
 * tq_w4a4_lr_gemm_a8_asym -- as tq_w4a4_lr_gemm_a8 with
 *   Y = bf16( s_w (s_x (acc + 8 wsum) + z_x wsum) + bf16(X L1) L2 ),
 *   acc = sum_k (q - 8) qw, so that acc + 8 wsum = sum_k q qw exactly.
 * Limits as tq_quantize_act_i8 / tq_w4a4_lr_gemm_a8; z_x and wsum 16-byte
 * aligned.
 */
TQ_API int tq_quantize_act_asym_i8(const uint16_t* X, int M, int K, int had_block,
                                   const uint16_t* L1t, int r, int8_t* Xq8, float* s_x,
                                   float* z_x, uint16_t* XL1b, void* stream);
TQ_API int tq_weight_code_sums(const uint8_t* Wq, int N, int K, int32_t* wsum, void* stream);
TQ_API int tq_w4a4_lr_gemm_a8_asym(const int8_t* Xq8, const float* s_x, const float* z_x,
                                   const uint8_t* Wq, const float* s_w, const int32_t* wsum,
                                   const uint16_t* XL1b, const uint16_t* L2t, int M, int N,
                                   int K, int r, uint16_t* Y, void* ws, size_t ws_bytes,
                                   void* stream);

/*
 * INT4 low-rank branch (TwinQuant notes section 04.C, Figure 4: both
 * components quantized).  The down projection reads the same rotated,
 * quantized activations as the residual GEMM: X L1 = (X H)(H^T L1) is
 * computed as the integer product of the activation codes with INT4 codes of
 * H^T L1 (per column j: scale s_L1[j]), dequantized with s_x s_L1 in fp32,
 * requantized per token to INT4 (symmetric, RoundClip, scale s_xl1), and fed
 * to a second integer product with INT4 codes of L2 (per output channel:
 * s_L2[n]); the shared epilogue adds s_xl1 s_L2 times that integer sum.
 *
 * tq_pack_lowrank_q4 -- offline: qL1 [r][K] s8, the codes of the rows of
 *   L1^T rotated like weight rows (had_block), one per byte (the factor is
 *   small and this is the tensor cores' operand layout), s_L1 [r]; qL2 [N][r]
 *   the codes of L2^T rows as bf16 integers, s_L2 [N].  r a multiple of 16,
 *   <= 512.
 * tq_quantize_act_qlr_i8 -- Xq8 [M][K] s8 codes and s_x [M] as
 *   tq_quantize_act_i8; XL1q [M][r] the requantized X L1 codes as bf16
 *   integers, s_xl1 [M].  The INT32 product runs on the tensor cores with K
 *   split over a thread-block cluster; the requantization is fused for r <=
 *   256.  Workspace >= tq_quantize_act_qlr_workspace_bytes (status word,
 *   INT32 scratch for wider ranks); a timeout is reported through
 *   tq_query_device_status on that workspace.
 * tq_w4a4_lr_gemm_a8_qlr -- Y = bf16( s_x s_w (Xq8 . Wq) +
 *   s_xl1 s_L2 (XL1q . qL2) ).  The second product runs on the bf16 MMA path
 *   with the integer codes: exact, since |code| <= 7 and |sum| <= 49 r < 2^24
 *   in the fp32 accumulator.
 */
TQ_API int tq_pack_lowrank_q4(const uint16_t* L1t, const uint16_t* L2t, int N, int K, int r,
                              int had_block, int8_t* qL1, float* s_L1, uint16_t* qL2,
                              float* s_L2, void* stream);
TQ_API size_t tq_quantize_act_qlr_workspace_bytes(int M, int K, int r);
TQ_API int tq_quantize_act_qlr_i8(const uint16_t* X, int M, int K, int had_block,
                                  const int8_t* qL1, const float* s_L1, int r, int8_t* Xq8,
                                  float* s_x, uint16_t* XL1q, float* s_xl1, void* workspace,
                                  size_t workspace_bytes, void* stream);
TQ_API int tq_w4a4_lr_gemm_a8_qlr(const int8_t* Xq8, const float* s_x, const uint8_t* Wq,
                                  const float* s_w, const uint16_t* XL1q, const float* s_xl1,
                                  const uint16_t* qL2, const float* s_L2, int M, int N, int K,
                                  int r, uint16_t* Y, void* ws, size_t ws_bytes, void* stream);

/*
 * tq_quantize_act_i8 -- tq_quantize_act for many tokens, with the codes one
 * per byte: the same rotation (CoQuant Eq. (3), block Hadamard), per-token
 * scale and RoundClip codes (CoQuant Eq. (1)) and the same X L1
 * (TwinQuant notes section 02.A), written for tq_w4a4_lr_gemm_a8.  tcgen05
 * has no dense int4 MMA kind, so the GEMM consumes int8 operands; codes in
 * int8 containers reach it without any unpacking (they are still INT4 values
 * in [-7, 7]).
 *
 *   X    [M][K] bf16    in : activations
 *   L1t  [r][K] bf16    in : L1^T; NULL iff r == 0
 *   Xq8  [M][K] s8     out : codes of X H, one per byte, in column order
 *   s_x  [M] fp32      out : per-token scales
 *   XL1b [M][r] bf16   out : bf16(X L1) (round to nearest even), the
 *                            low-rank GEMM operand; NULL iff r == 0
 * Limits: had_block <= 128 (else TQ_ERR_UNSUPPORTED_SHAPE).  Ranks above 128
 * run the codes and X L1 as separate launches (X L1 in launches of at most
 * 256 columns) on the same stream.
 */
TQ_API int tq_quantize_act_i8(const uint16_t* X, int M, int K, int had_block,
                              const uint16_t* L1t, int r,
                              int8_t* Xq8, float* s_x, uint16_t* XL1b, void* stream);

/*
 * tq_w4a4_lr_gemm_a8 -- tq_w4a4_lr_gemm with the activation codes one per
 * byte (from tq_quantize_act_i8):
 *
 *   Y[m][n] = bf16( s_x[m] s_w[n] sum_k qx[m][k] qw[n][k]
 *                   + sum_j XL1b[m][j] L2t[n][j] )
 *
 * the integer sum exact in INT32.  Workspace: at least
 * tq_gemm_workspace_bytes bytes, zeroed before first use.  With at least
 * tq_gemm_a8_workspace_bytes bytes (a ~16 MB scratch after the status word)
 * and a tile count that is not a whole multiple of the SM count, the
 * persistent CTAs split the tiles x k-blocks evenly (stream-K): a CTA that
 * computes part of a tile another CTA finishes leaves its INT32 partial sums
 * and ready flags in the scratch, and the finishing CTA clears the flags, so
 * the scratch is zero again after every call that completes.  Y is the same
 * bit for bit under either schedule (integer sums).  After a call whose
 * status reports TQ_ERR_TIMEOUT, zero the workspace again.  Calls that share
 * a workspace must not overlap.  tq_w4a4_lr_gemm_a8_asym, ..._qlr, the layer
 * (M > 128) and tq_w4a4_lr_gate_up follow the same rule with their own
 * workspace sizes.
 */
TQ_API size_t tq_gemm_a8_workspace_bytes(int M, int N, int K, int r);
TQ_API int tq_w4a4_lr_gemm_a8(const int8_t* Xq8, const float* s_x,
                              const uint8_t* Wq, const float* s_w,
                              const uint16_t* XL1b, const uint16_t* L2t,
                              int M, int N, int K, int r, uint16_t* Y,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * tq_debug_w4a4_gemm_acc -- test hook: the same GEMM kernel with the
 * low-rank branch off, writing the raw INT32 accumulators
 * acc[m][n] = sum_k qx[m][k] qw[n][k] to `acc` [M][N] (int32) instead of Y.
 * Lets a caller check the integer path bit-exactly on codes of its choice.
 */
TQ_API int tq_debug_w4a4_gemm_acc(const uint8_t* Xq, const uint8_t* Wq,
                           int M, int N, int K, int32_t* acc,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * tq_w4a4_lr_gemm_noalloc -- tq_w4a4_lr_gemm for callers that cannot
 * allocate device memory (a framework that owns the device allocator, a
 * real-time path where an allocation could synchronise the device, a plugin
 * that only ever receives pointers to its inputs and outputs).  Same inputs,
 * output and result as tq_w4a4_lr_gemm, but no workspace argument: the
 * kernel's scratch (its status word) lives in a fixed 256-byte array in the
 * library's own device memory, which every GPU that loads the library keeps
 * until the process exits.  Nothing is allocated on any call.
 *
 *  - Argument errors are returned before any device work, in the same order
 *    as tq_w4a4_lr_gemm.  Shapes needing more scratch than
 *    tq_gemm_workspace_bytes() = 256 bytes are rejected with
 *    TQ_ERR_WORKSPACE.
 *  - The first call in a CUDA context looks up that array's device address
 *    (with that context current) and caches it per context; make that first
 *    call before any stream capture.
 *  - Every call shares the array, which keeps what the last call left in it.
 *    Nothing in it needs to start at zero for the result: the kernel writes
 *    only the status word, and only when a bounded wait gives up.  Calls that
 *    overlap on the GPU (different streams with no ordering between them)
 *    race on it.
 *  - tq_noalloc_query_status(stream) synchronises `stream`, then reads and
 *    clears that status word: TQ_OK, or TQ_ERR_TIMEOUT if a bounded wait of
 *    any no-allocation call in this context gave up since the last query.
 *  - tq_debug_noalloc_set_status(status) is a test hook: it writes `status`
 *    into that word (synchronously, no kernel).
 * The pages have no counterpart of this entry point; it is an addition of
 * this library.
 */
TQ_API int tq_w4a4_lr_gemm_noalloc(const uint8_t* Xq, const float* s_x,
                                   const uint8_t* Wq, const float* s_w,
                                   const float* XL1, const uint16_t* L2t,
                                   int M, int N, int K, int r, uint16_t* Y,
                                   void* stream);
TQ_API int tq_noalloc_query_status(void* stream);
TQ_API int tq_debug_noalloc_set_status(int status);

/*
 * tq_debug_w4a4_lr_layer_decode -- test hook: the one-kernel decode layer of
 * tq_w4a4_lr_layer (M <= 16, r in {0, 16, 32, 64}, K % 256 == 0, K <= 4096,
 * had_block <= 256), also writing what it computes on the way: the
 * activation codes `codes` [M][K] int8 (RoundClip of X H per token), the
 * scales `s_x` [M] fp32 and the integer sums `acc` [M][N] int32
 * (sum_k codes[m][k] qw[n][k], exact).  Each of the three may be NULL.
 * Shapes the kernel does not serve return TQ_ERR_UNSUPPORTED_SHAPE.
 */
TQ_API int tq_debug_w4a4_lr_layer_decode(const uint16_t* X, const uint16_t* L1t,
                                         const uint8_t* Wq, const float* s_w,
                                         const uint16_t* L2t, int M, int N, int K, int r,
                                         int had_block, uint16_t* Y, int8_t* codes, float* s_x,
                                         int32_t* acc, void* workspace, size_t workspace_bytes,
                                         void* stream);

/*
 * tq_debug_watchdog -- test hook for the bounded waits every pipelined
 * kernel here uses.  Launches one CTA (no cluster) in which a producer lane
 * arrives on an mbarrier, unless `withhold` is non-zero, and a consumer lane
 * waits for that arrival with the library's bounded wait, giving up after
 * `budget_cycles` SM cycles (1000 .. 2e9).  A wait that gives up writes
 * TQ_ERR_TIMEOUT into the status word at the start of `workspace` (>= 256
 * bytes, a GEMM workspace), read back by tq_query_device_status; the kernel
 * then returns normally and the context stays usable.  *waited_ok (a device
 * int) is set to 1 when the arrival was seen, 0 when the wait gave up.
 * No counterpart on the pages: it tests the library's own failure handling.
 */
TQ_API int tq_debug_watchdog(void* workspace, size_t workspace_bytes, int withhold,
                             long long budget_cycles, int* waited_ok, void* stream);

/*
 * tq_query_device_status -- synchronises `stream`, then reads the status word
 * kernels record in `workspace` (a GEMM workspace) and clears it.  Returns
 * TQ_OK, TQ_ERR_TIMEOUT if a bounded in-kernel wait gave up since the last
 * query, or TQ_ERR_CUDA.
 */
TQ_API int tq_query_device_status(void* workspace, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H_ */
