/*
 * bsq.h -- libbsq: block-scaled quantization (NVFP4, MXFP8, MXFP4), the 16-point
 * random Hadamard transform and block-scaled GEMMs for NVIDIA B200
 * (sm_100a).  Plain C ABI: device pointers, sizes, a stream handle.
 *
 * Formats (web pages cited by title and section):
 *  - NVFP4 -- "Microscaling (MX) and block-scaled 4-bit formats", section
 *    "NVFP4"; "08 -- FP4, MXFP4, NVFP4: The Blackwell Frontier", table "The
 *    two Blackwell formats": E2M1 elements in blocks of 16, one E4M3 scale
 *    per block, one FP32 per-tensor scale.  Codes are packed two per byte,
 *    element 2j in the low nibble of byte j.
 *  - MXFP8 -- "LMSYS and humans& ... low-precision recipes", section "Recipe
 *    1: End-to-end MXFP8": 32 consecutive E4M3 share one E8M0 scale.
 *  - MXFP4 -- "08 -- FP4, MXFP4, NVFP4 ...", table "The two Blackwell
 *    formats": 32 consecutive E2M1 share one E8M0 scale (4.25 bits).
 *  - Scale-factor ("SF") buffers are written in the layout the Blackwell
 *    block-scaled MMA reads ("Microscaling ...", section "Hardware and
 *    kernels": a block-scaled GEMM needs a particular scale-factor layout):
 *    128-row x 4-block atoms of 512 bytes; row r, block b of an atom sits at
 *    byte (r % 32) * 16 + (r / 32) * 4 + b; atoms are ordered row-tile major,
 *    then block tile; rows pad to 128 and blocks to 4.  bsq_sf_bytes() gives
 *    the size.  Padding bytes are never written by the quantizers.
 *
 * Conventions for every entry point:
 *  - Pointers named *_dev, and all tensor pointers, are DEVICE pointers on
 *    the current device, allocated and owned by the caller; none is retained
 *    after the call returns.  Tensor pointers must be 16-byte aligned.
 *  - bf16 matrices are row-major with a leading dimension in elements (ld*),
 *    which must be a multiple of 8.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *    only enqueues work on it: it never synchronizes and returns a bsq status
 *    from host-side argument validation alone (an invalid call launches
 *    nothing).  Faults found on the device (a bounded wait that ran out) are
 *    recorded in a per-device error word that bsq_check() reads.
 *  - The library allocates no device memory on these paths except, once per
 *    device, the 4-byte error word (created on first use).
 *  - Inputs must be finite; nonzero magnitudes below 2^-100 are outside the
 *    supported range for NVFP4 (codes there are unspecified).
 *  - Behaviour is selected by the arguments alone; the library reads no
 *    environment variable.  bsq_debug_kernel_choice() can force one of two
 *    equivalent kernels for tests and tuning (results are identical).
 *  - CUDA graphs: the quantize and GEMM entry points may be called on a
 *    stream under capture once the same calls have run once outside capture
 *    on that device (the first call creates the per-device error word and
 *    sets kernel attributes).  Under capture an amax + quantize pair is
 *    recorded as two ordinary kernels instead of one cooperative launch;
 *    the bytes are the same.  The GEMM's tensor maps are encoded at call
 *    time from the pointers given, so a replayed graph uses those buffers.
 *    bsq_check() synchronizes and may not be called under capture.
 */
#ifndef BSQ_H
#define BSQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BSQ_API __attribute__((visibility("default")))
#else
#define BSQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum {
    BSQ_OK = 0,
    BSQ_ERR_INVALID = 1,     /* bad size, null pointer or option mix */
    BSQ_ERR_ALIGN = 2,       /* pointer or leading dimension misaligned */
    BSQ_ERR_UNSUPPORTED = 3, /* valid request the library does not handle */
    BSQ_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed */
    BSQ_ERR_TIMEOUT = 5      /* a device-side bounded wait ran out */
};

enum { BSQ_RNE = 0, BSQ_SR = 1 };          /* rounding for MXFP8 outputs */
enum { BSQ_NVFP4 = 0, BSQ_MXFP8 = 1, BSQ_MXFP4 = 2 }; /* GEMM operand format */
enum { BSQ_OUT_F32 = 0, BSQ_OUT_BF16 = 1 }; /* GEMM output type */

/* Kernel-selection overrides (bsq_debug_kernel_choice). */
enum {
    BSQ_KNOB_FUSED_QUANT = 0, /* 1/-1: amax + 16x16 quantize in one cooperative launch; 0: two passes */
    BSQ_KNOB_GEMM_PAIR = 1,   /* -1: automatic; 0: single-CTA GEMM; 1: CTA-pair GEMM where it applies */
    BSQ_KNOB_GEMM_BN = 2,     /* -1: automatic; 128 or 256 (bf16 output): the single-CTA GEMM's N tile */
    BSQ_KNOB_STREAM_QUANT = 3, /* -1: bulk-copy streaming NVFP4 kernels for contiguous 16x16 tensors; 1: for every
                                  contiguous amax / NVFP4 call; 0: never */
    BSQ_KNOB_GEMM_SPLITK = 4,  /* -1: automatic; 1: off; 2, 4 or 8: the skinny (M <= 64) GEMM's K split */
    BSQ_KNOB_LAUNCH_OVERLAP = 5 /* 1/-1: the GEMMs and the linear step's quantize kernels are launched for
                                   programmatic dependent launch (scheduled while the previous kernel in the
                                   stream finishes; each waits for it before touching memory); 0: plain launches */
};

/* Human-readable name of a status code (static string). */
BSQ_API const char *bsq_status_str(int status);

/* Bytes of a swizzled scale-factor buffer for `rows` rows of `nblocks`
 * blocks: roundup(rows,128) * roundup(nblocks,4).  Host-only helper. */
BSQ_API size_t bsq_sf_bytes(int64_t rows, int64_t nblocks);

/* RHT sign vector for a seed: bits 0..15 of word 0 of Philox4x32-10 with
 * counter 0 and key (lo32(seed), hi32(seed)) (Salmon et al., SC'11); bit i
 * set means s_i = -1.  Host-only helper, no device work. */
BSQ_API uint16_t bsq_rht_sign_mask(uint64_t seed);

/* Tensor amax: *amax_dev = max |x| over the M x K bf16 matrix x (rows
 * selected through row_index[0..M) when it is not NULL), after the 16-point
 * RHT along K when rht_enable != 0 (see bsq_rht).  This is the first level of
 * NVFP4's two-level scale ("Microscaling ...", section "NVFP4").
 * K % 16 == 0.  *amax_dev is overwritten (zeroed on the stream first). */
BSQ_API int bsq_amax(const void *x_bf16, int64_t M, int64_t K, int64_t ldx,
             int rht_enable, uint16_t rht_sign_mask, const int32_t *row_index_dev,
             float *amax_dev, void *stream);

/* The NVFP4 global scale s_g = amax / 2688 (amax = 0 gives 1) of the M x K
 * bf16 matrix x, after the 16-point RHT along K when rht_enable != 0 -- the
 * value bsq_quant_nvfp4 writes to *global_scale_dev -- computed without
 * allocating any device memory.  The pages have no counterpart to this
 * entry point.  It is for callers that may not call cudaMalloc: code whose
 * device memory all belongs to a framework's pool allocator (a raw
 * allocation would sit outside the pool's accounting and cap), and code on
 * a latency-critical path, where cudaMalloc can synchronize the device.
 * Its scratch is a file-scope device array of 16 KiB (4096 words) that every
 * GPU which loads the library holds until the process exits: word 0 counts
 * finished CTAs, word 1 + c holds CTA c's maximum, one CTA per 65536
 * elements.  A request needing more (M * K > 4095 * 65536 elements, about
 * 268 million) returns BSQ_ERR_UNSUPPORTED without touching the device.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call
 * outside any stream capture.  Each call zeroes the counter on the stream
 * before its kernel.  All calls on one device share the array, which keeps
 * the last call's contents: calls that overlap on the GPU race, so order
 * them on one stream or synchronize between them.  Never allocates, not even
 * the error word of the other entry points.  K % 16 == 0; x 16-byte aligned,
 * ldx % 8 == 0; gs_dev 4-byte aligned. */
BSQ_API int bsq_global_scale_noalloc(const void *x_bf16, int64_t M, int64_t K, int64_t ldx, int rht_enable,
                                     uint16_t rht_sign_mask, float *gs_dev, void *stream);

/* NVFP4 quantize ("Microscaling ...", section "NVFP4"; "Thinking Machines
 * ... Inkling 2 Small", section "A precision choice for each stage" for Four
 * Over Six).  Output row i is input row row_index[i] (or i when row_index is
 * NULL); with rht_enable the 16-point RHT along K is applied first (fp32).
 *   s_g = amax / 2688 (amax = 0 gives s_g = 1); amax is *amax_in_dev, or is
 *         computed here when amax_in_dev is NULL (an amax pass that uses
 *         the first 8 bytes of codes as its scratch before the quantize
 *         pass overwrites them);
 *   per block (1x16 along K, or a 16x16 tile with block_2d):
 *         s_b = E4M3_RNE((block_amax / 6) / s_g), r = 1 / (s_b * s_g),
 *         code = E2M1_RNE_sat(x * r); s_b == 0 gives all-zero codes;
 *   four_over_six (1x16 only): also try block_amax / 4 and keep it when its
 *         squared error (pairwise fp32 sum over the 16 elements) is lower.
 * Outputs: *global_scale_dev = s_g; codes [M][K/2] bytes (row stride K/2);
 * sf swizzled.  With G > 0 the rows form G groups (MoE experts): group e
 * owns output rows [row_offsets[e], row_offsets[e+1]) and its SF rows start
 * at sf_row_offsets[e] (a multiple of 128); both arrays are device int32
 * [G+1], nondecreasing, with row_offsets[0] = 0 and row_offsets[G] = M, and
 * sf must hold sf_row_offsets[G] SF rows (a row outside [row_offsets[0],
 * row_offsets[G]) gets codes but writes no scale factor).
 * Requirements: K % 16 == 0; block_2d needs M % 16 == 0 and excludes
 * four_over_six and groups. */
BSQ_API int bsq_quant_nvfp4(const void *x_bf16, int64_t M, int64_t K, int64_t ldx,
                    int block_2d, int four_over_six, int rht_enable, uint16_t rht_sign_mask,
                    const int32_t *row_index_dev,
                    int G, const int32_t *row_offsets_dev, const int32_t *sf_row_offsets_dev,
                    const float *amax_in_dev, float *global_scale_dev,
                    uint8_t *codes_dev, uint8_t *sf_dev, void *stream);

/* NVFP4 quantize of gathered rows, for gathers that repeat rows (MoE
 * routing sends each token to several experts).  The result is byte for
 * byte that of bsq_quant_nvfp4 with the same row_index (1x16 blocks,
 * optional Four Over Six and RHT, expert groups, amax_in semantics): output
 * row i is the quantization of source row row_index[i] under the global
 * scale of the gathered rows' amax.  Since a row's codes and scales depend
 * only on its source row and s_g, the T source rows (x is [T][K]) are
 * quantized once into the caller's workspace and then moved to the output
 * rows.  workspace: device memory of at least
 * bsq_quant_nvfp4_gather_workspace(T, K) bytes, 256-byte aligned, owned by
 * the caller (its contents are scratch); every row_index value must be in
 * [0, T).  K % 64 == 0.  G <= 1024 (BSQ_ERR_UNSUPPORTED above). */
BSQ_API size_t bsq_quant_nvfp4_gather_workspace(int64_t T, int64_t K);
BSQ_API int bsq_quant_nvfp4_gather(const void *x_bf16, int64_t T, int64_t K, int64_t ldx,
                                   const int32_t *row_index_dev, int64_t M, int four_over_six, int rht_enable,
                                   uint16_t rht_sign_mask, int G, const int32_t *row_offsets_dev,
                                   const int32_t *sf_row_offsets_dev, const float *amax_in_dev,
                                   float *global_scale_dev, uint8_t *codes_dev, uint8_t *sf_dev, void *workspace_dev,
                                   size_t workspace_bytes, void *stream);

/* NVFP4 quantize with stochastic rounding of the elements ("Microscaling
 * ...", section "NVFP4": the NVFP4 pretraining recipe rounds gradients
 * stochastically).  s_g, the block scales (1x16, or 16x16 with block_2d)
 * and the scratch use are those of bsq_quant_nvfp4; each element
 * q = y * r (y the RHT output when rht_enable, r = 1 / (s_b * s_g)) is
 * clamped to +-6 and rounded to a neighbouring E2M1 value: up iff
 * draw * 2^-16 < (|q| - lo) / (hi - lo), with the 16-bit draws of
 * bsq_quant_mxfp8 for output element idx = row * K + k.  s_b == 0 gives
 * all-zero codes.  Optional row gather (row_index_dev, 1x16 only); no Four
 * Over Six and no expert groups.  K % 16 == 0; block_2d needs M % 16 == 0. */
BSQ_API int bsq_quant_nvfp4_sr(const void *x_bf16, int64_t M, int64_t K, int64_t ldx, int block_2d,
                       int rht_enable, uint16_t rht_sign_mask, const int32_t *row_index_dev,
                       const float *amax_in_dev, float *global_scale_dev, uint64_t seed,
                       uint32_t stream_id, uint8_t *codes_dev, uint8_t *sf_dev, void *stream);

/* MXFP8 quantize ("LMSYS and humans& ...", section "Recipe 1"; stochastic
 * rounding per "Microscaling ...", section "Words on this page", and
 * "Thinking Machines ...", section "A precision choice for each stage").
 * Per block of 32: E = clamp(floor(log2 block_amax) - 8, -127, 127), scale
 * code E + 127 (an all-zero block has code 0); element x * 2^-E clamped to
 * +-448, then E4M3 by nearest-even (BSQ_RNE) or stochastic rounding
 * (BSQ_SR) with 16-bit draws from Philox4x32-10: the output element with
 * row-major index idx (in the OUTPUT shape) uses counter (lo32(idx>>3),
 * hi32(idx>>3), stream_id, 0), key (lo32(seed), hi32(seed)), and the low
 * (idx even) or high (idx odd) half of word (idx>>1)&3; it rounds up iff
 * draw * 2^-16 < the fractional position between the two neighbours.
 * colwise == 0: blocks along K, codes [M][K], sf for M rows x K/32 blocks.
 * colwise == 1: the quantization of x^T -- codes [K][M] (row stride M), sf
 * for K rows x M/32 blocks.  K % 32 == 0 (row-wise); M % 32 == 0 and
 * K % 8 == 0 (column-wise).  Column-wise tensors with
 * (M / 32) * ceil(K / 64) >= 2^31 return BSQ_ERR_UNSUPPORTED. */
BSQ_API int bsq_quant_mxfp8(const void *x_bf16, int64_t M, int64_t K, int64_t ldx, int colwise,
                    int rounding, uint64_t seed, uint32_t stream_id,
                    uint8_t *codes_dev, uint8_t *sf_dev, void *stream);

/* Row-wise and column-wise MXFP8 of one bf16 matrix in a single pass
 * ("Thinking Machines ...", section "A precision choice for each stage": the
 * backward pass consumes gradients in MXFP8 with stochastic rounding, along
 * both of dY's axes).  The outputs are exactly those of bsq_quant_mxfp8 with
 * colwise = 0 (stream id stream_id_row) and colwise = 1 (stream id
 * stream_id_col), same seed and rounding: codes_row [M][K] with sf_row for
 * M rows x K/32 blocks, codes_col [K][M] with sf_col for K rows x M/32
 * blocks; x is read once.  M % 32 == 0 and K % 32 == 0;
 * (M / 32) * ceil(K / 64) >= 2^31 returns BSQ_ERR_UNSUPPORTED. */
BSQ_API int bsq_quant_mxfp8_rowcol(const void *x_bf16, int64_t M, int64_t K, int64_t ldx, int rounding,
                                   uint64_t seed, uint32_t stream_id_row, uint32_t stream_id_col,
                                   uint8_t *codes_row_dev, uint8_t *sf_row_dev, uint8_t *codes_col_dev,
                                   uint8_t *sf_col_dev, void *stream);

/* NVFP4 -> MXFP8 column-wise requantize ("Thinking Machines ...", section
 * "A precision choice for each stage": tensors saved in NVFP4 during the
 * forward pass -- the weights in 16x16 blocks -- are dequantized, transposed
 * at higher precision and requantized to MXFP8 for the backward pass).  The
 * NVFP4 matrix [R][C] (codes [R][C/2], swizzled E4M3 scales for R rows x
 * C/16 blocks as bsq_quant_nvfp4 writes them, *gs_dev its FP32 global scale)
 * is decoded to fp32 as RN(RN(E2M1 * s_b) * s_g) (the first product is
 * exact), transposed, and quantized as bsq_quant_mxfp8 does: blocks of 32
 * along R, element idx = c * R + r for the stochastic draws.  Outputs
 * codes_col [C][R], sf_col for C rows x R/32 blocks.  R % 32 == 0,
 * C % 16 == 0; (R / 32) * ceil(C / 64) >= 2^31 returns BSQ_ERR_UNSUPPORTED. */
BSQ_API int bsq_requant_nvfp4_mxfp8(const uint8_t *codes_dev, const uint8_t *sf_dev, const float *gs_dev,
                                    int64_t R, int64_t C, int rounding, uint64_t seed, uint32_t stream_id,
                                    uint8_t *codes_col_dev, uint8_t *sf_col_dev, void *stream);

/* MXFP4 quantize ("08 -- FP4, MXFP4, NVFP4 ...", section "The two Blackwell
 * formats": E2M1 elements in groups of 32 with one E8M0 power-of-two scale,
 * 4.25 bits per value; "Microscaling ...", section "Microscaling").  Per
 * row-wise block of 32: E = clamp(floor(log2 block_amax) - 2, -127, 127)
 * (2 is the exponent of E2M1's largest value 6 = 1.5 * 2^2, as 8 is E4M3's
 * for MXFP8), scale code E + 127 (an all-zero block has code 0 and +0
 * codes); element x * 2^-E clamped to +-6, then E2M1 by nearest-even
 * (BSQ_RNE) or stochastic rounding (BSQ_SR) with the draws of
 * bsq_quant_mxfp8 (output element idx = row * K + k).  codes [M][K/2],
 * element 2j in the low nibble of byte j; sf in the swizzled MMA layout for
 * M rows x K/32 blocks.  K % 32 == 0; x, codes, sf 16-byte aligned,
 * ldx % 8 == 0. */
BSQ_API int bsq_quant_mxfp4(const void *x_bf16, int64_t M, int64_t K, int64_t ldx, int rounding,
                    uint64_t seed, uint32_t stream_id, uint8_t *codes_dev, uint8_t *sf_dev,
                    void *stream);

/* 16-point random Hadamard transform along K ("Microscaling ...", section
 * "NVFP4"; "Thinking Machines ...", section "Why communication became the
 * next bottleneck"): per group of 16, y = 1/4 * H16 * diag(s) * x with H16
 * the Sylvester Hadamard matrix, computed in fp32 by butterflies of stride
 * 1, 2, 4, 8 and rounded to bf16 (nearest-even).  K % 16 == 0.  x and y may
 * not overlap unless they are the same buffer with the same ld. */
BSQ_API int bsq_rht(const void *x_bf16, void *y_bf16, int64_t M, int64_t K, int64_t ldx, int64_t ldy,
            uint16_t rht_sign_mask, void *stream);

/* Block-scaled S2F6 for the MoE combine exchange ("Thinking Machines ...",
 * section "Why communication became the next bottleneck": expert outputs
 * are rotated by a random Hadamard transform and sent in block-scaled S2F6,
 * an 8-bit fixed-point format, at 8.25 bits per value).  S2F6 is read here
 * as two's-complement fixed point with six fraction bits: code q in
 * [-128, 127] stands for q / 64.  Per row, after the 16-point RHT along K
 * when rht_enable != 0 (as bsq_rht, in fp32): each block of 32 has one
 * E8M0 scale code E + 127 with E = clamp(floor(log2 block_amax), -127, 127)
 * (an all-zero block: code 0 and zero codes), and q = nearest-even integer
 * of x * 2^(6 - E), clamped to [-128, 127].  codes [M][K] int8 (row stride
 * K), sf [M][K/32] bytes row-major.  K % 32 == 0; x and codes 16-byte
 * aligned, ldx % 8 == 0. */
BSQ_API int bsq_quant_s2f6(const void *x_bf16, int64_t M, int64_t K, int64_t ldx, int rht_enable,
                           uint16_t rht_sign_mask, int8_t *codes_dev, uint8_t *sf_dev, void *stream);

/* The S2F6 receiver (same page and section: the receiver reconstructs and
 * combines the values, then reverses the transform).  For token t, the rows
 * rows_dev[token_offsets_dev[t] .. token_offsets_dev[t+1]) of the S2F6
 * matrix (codes [R][K], sf [R][K/32] as bsq_quant_s2f6 writes them) are
 * decoded (q / 64 * 2^E, exact) and summed in list order with the weights
 * weights_dev[j] (fp32: one rounding per product and per addition); each
 * group of 16 of the sum is then rotated back, x = 1/4 * D * H16 * acc (the
 * inverse of bsq_rht's transform with the same sign mask), and rounded to
 * bf16: out [T][K] with leading dimension ldo.  token_offsets_dev is int32
 * [T+1], rows_dev int32 and weights_dev fp32 of its last value's length.
 * K % 32 == 0; codes and out 16-byte aligned, ldo % 8 == 0. */
BSQ_API int bsq_combine_s2f6(const int8_t *codes_dev, const uint8_t *sf_dev, int64_t K,
                             const int32_t *token_offsets_dev, const int32_t *rows_dev, const float *weights_dev,
                             int64_t T, uint16_t rht_sign_mask, void *out_bf16_dev, int64_t ldo, void *stream);

/* Byte movers for the expert-parallel exchange (the pages describe the
 * dispatch of NVFP4 rows to the GPUs holding the experts and the combine
 * back, "Thinking Machines ...", section "Why communication became the next
 * bottleneck"; these calls do no arithmetic).
 * bsq_gather_rows: dst row r = src row index_dev[r], rows of row_bytes
 * bytes (a multiple of 16); src and dst 16-byte aligned.
 * bsq_sf_to_rows: a swizzled scale-factor buffer (rows x nblk blocks, as
 * the quantizers write it) to plain rows of nblk bytes.
 * bsq_sf_from_rows: plain rows back into the swizzled layout; with G > 0,
 * row r of group e (device int32 offsets as for bsq_quant_nvfp4) goes to SF
 * row r - row_offsets[e] + sf_row_offsets[e] (the grouped GEMM's layout).
 * Padding bytes of the swizzled buffer are not written.  Both take
 * rows * nblk < 2^31 (BSQ_ERR_UNSUPPORTED above). */
BSQ_API int bsq_gather_rows(const void *src_dev, int64_t row_bytes, const int32_t *index_dev, int64_t R,
                            void *dst_dev, void *stream);
BSQ_API int bsq_sf_to_rows(const uint8_t *sf_dev, int64_t rows, int64_t nblk, uint8_t *rows_out_dev, void *stream);
BSQ_API int bsq_sf_from_rows(const uint8_t *rows_in_dev, int64_t rows, int64_t nblk, int G,
                             const int32_t *row_offsets_dev, const int32_t *sf_row_offsets_dev, uint8_t *sf_dev,
                             void *stream);

/* Dequantize -> transpose -> requantize ("Thinking Machines ...", section
 * "A precision choice for each stage"): the row-wise MXFP8 tensor (codes
 * [M][K], swizzled sf for M x K/32) is decoded exactly (E4M3 x 2^E, fp32),
 * transposed, and quantized again as in bsq_quant_mxfp8 with blocks of 32
 * along the old M: codes_col [K][M], sf_col for K rows x M/32 blocks.
 * M % 32 == 0 and K % 32 == 0 (whole blocks of 32 along both axes);
 * (M / 32) * ceil(K / 64) >= 2^31 returns BSQ_ERR_UNSUPPORTED. */
BSQ_API int bsq_requant_transpose(const uint8_t *codes_row_dev, const uint8_t *sf_row_dev,
                          int64_t M, int64_t K, int rounding, uint64_t seed, uint32_t stream_id,
                          uint8_t *codes_col_dev, uint8_t *sf_col_dev, void *stream);

/* Block-scaled GEMM ("Microscaling ...", section "Hardware and kernels":
 * the tensor core applies the block scales inside the matrix instruction):
 *   C[m][n] = alpha * sum_k decA[m][k] * decB[n][k],
 * A [M][K] and B [N][K] both K-major (codes row-major, as the quantizers
 * write them), with their swizzled SF buffers.  NVFP4: alpha =
 * (*gsA_dev) * (*gsB_dev) (each may be NULL for 1); MXFP8 and MXFP4 (E2M1
 * codes packed as bsq_quant_mxfp4 writes them, one E8M0 scale per 32
 * elements; "08 -- FP4, MXFP4, NVFP4 ...", table "The two Blackwell
 * formats"): alpha = 1 and gs* are ignored.  Accumulation is fp32 in tensor memory; C is fp32 or
 * bf16 (nearest-even), row-major with leading dimension ldc (elements).
 * Requirements: K % 128 == 0; M, N >= 1. */
BSQ_API int bsq_gemm_blockscaled(int fmt, const uint8_t *A_dev, const uint8_t *sfA_dev, const float *gsA_dev,
                         const uint8_t *B_dev, const uint8_t *sfB_dev, const float *gsB_dev,
                         int64_t M, int64_t N, int64_t K, void *C_dev, int64_t ldc, int out_type,
                         void *stream);

/* Grouped block-scaled GEMM for MoE experts ("Thinking Machines ...",
 * section "A precision choice for each stage": NVFP4 forward in the
 * expert layers).  For each group e with rows [row_offsets[e],
 * row_offsets[e+1]) of A (M_total rows in all):
 *   C[m][n] = alpha_e * sum_k decA[m][k] * decB_e[n][k],
 * alpha_e = (*gsA_dev) * gsB_dev[e] for NVFP4 (either may be NULL for 1).
 * A's SF rows of group e start at sf_row_offsets[e] (as bsq_quant_nvfp4
 * writes them with groups); B is [G][N][K] codes with G consecutive SF
 * buffers of bsq_sf_bytes(N, K/vec) bytes each.  Offsets are device int32
 * [G+1], nondecreasing, row_offsets[0] = 0 and row_offsets[G] <= M_total
 * (no row of C past M_total is written); the row counts may be anything
 * (zero included).  K % 128 == 0. */
BSQ_API int bsq_grouped_gemm(int fmt, int G, const int32_t *row_offsets_dev, const int32_t *sf_row_offsets_dev,
                     int64_t M_total, const uint8_t *A_dev, const uint8_t *sfA_dev, const float *gsA_dev,
                     const uint8_t *B_dev, const uint8_t *sfB_dev, const float *gsB_dev,
                     int64_t N, int64_t K, void *C_dev, int64_t ldc, int out_type, void *stream);

/* Grouped NVFP4 GEMM whose output is written in NVFP4 ("Microscaling ...",
 * section "Open points": fused quantize-and-GEMM kernels, since computing
 * block scales is itself memory traffic; "Thinking Machines ...", section
 * "Why communication became the next bottleneck": kernels that combine
 * matrix operations, quantization and rounding).  The MoE up projection's
 * output H feeds the down projection in NVFP4, so the epilogue quantizes it
 * directly instead of storing bf16 H and reading it back: for each group
 * e, H[m][n] = bf16_RNE(alpha_e * sum_k decA[m][k] decB_e[n][k]) exactly as
 * bsq_grouped_gemm computes it, then NVFP4 with 1x16 blocks as
 * bsq_quant_nvfp4 computes it -- Four Over Six when four_over_six != 0 --
 * but with the GIVEN global scale *out_gs_dev (a tensor scale must be known
 * before the first block is quantized, and the GEMM produces H tile by
 * tile: the caller passes a scale from an earlier amax, e.g. the previous
 * step's, as delayed scaling does).  Outputs: out_codes [M_total][N/2];
 * out_sf swizzled for N/16 blocks per row, group e's rows starting at SF row
 * sf_row_offsets[e] (the layout bsq_grouped_gemm reads for A); *out_amax_dev
 * (if not NULL; zeroed first) = max |H| over all rows, from which the next
 * global scale amax / 2688 follows.  C_bf16_dev, if not NULL, also receives
 * H in bf16 (leading dimension ldc).  Operands as for bsq_grouped_gemm with
 * fmt = BSQ_NVFP4 (other formats: BSQ_ERR_UNSUPPORTED); N % 64 == 0,
 * N >= 128, K % 256 == 0. */
BSQ_API int bsq_grouped_gemm_nvfp4_out(int fmt, int G, const int32_t *row_offsets_dev,
                                       const int32_t *sf_row_offsets_dev, int64_t M_total, const uint8_t *A_dev,
                                       const uint8_t *sfA_dev, const float *gsA_dev, const uint8_t *B_dev,
                                       const uint8_t *sfB_dev, const float *gsB_dev, int64_t N, int64_t K,
                                       const float *out_gs_dev, int four_over_six, uint8_t *out_codes_dev,
                                       uint8_t *out_sf_dev, float *out_amax_dev, void *C_bf16_dev, int64_t ldc,
                                       void *stream);

/* Synchronize `stream`, then read and clear this device's error word.
 * Returns BSQ_OK, BSQ_ERR_TIMEOUT (a kernel's bounded wait ran out; the
 * kernel returned early and its outputs are undefined) or BSQ_ERR_CUDA. */
BSQ_API int bsq_check(void *stream);

/* Forces a kernel choice (BSQ_KNOB_* with the values listed there; -1
 * restores the automatic choice) for every later call in this process, on
 * every device.  Host-only and thread-safe; results are bit-identical either
 * way -- it exists so that tests and timing can reach each kernel.  Returns
 * BSQ_ERR_INVALID for an unknown knob or value. */
BSQ_API int bsq_debug_kernel_choice(int knob, int value);

/* Test hook for the bounded-wait path: launches one CTA that waits on a
 * shared-memory barrier nobody arrives at, giving up after timeout_ns
 * nanoseconds (device clock) and recording BSQ_ERR_TIMEOUT.  The context
 * stays usable.  timeout_ns must be in (0, 10^10]. */
BSQ_API int bsq_debug_timeout_probe(uint64_t timeout_ns, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* BSQ_H */
