// quant.cuh -- host-side launchers of the codec kernels (quant.cu).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace bsq {

// amax into *amax_bits (zeroed by the caller).  With a counter (zeroed by
// the caller too) the kernel's last CTA also writes s_g = amax / 2688 to
// *gs_out.
void launch_amax(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, bool rht, uint32_t mask,
                 const int32_t *row_index, unsigned int *amax_bits, unsigned int *counter, float *gs_out,
                 int num_sms, cudaStream_t s);
void launch_finalize_global_scale(float *gs, cudaStream_t s);
// 16-element blocks per CTA of the partial-maximum amax pass.
constexpr int kPartialBlocks = 4096;
// amax + s_g with one partial maximum per CTA in `scratch`: word 0 is a CTA
// counter (zero on entry), words 1 .. ceil(M K / 16 / kPartialBlocks) hold
// the partials.  The last CTA writes s_g to *gs_out.
void launch_amax_partials(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, bool rht, uint32_t mask,
                          unsigned int *scratch, float *gs_out, cudaStream_t s);
void launch_quant_nvfp4(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, bool block_2d, bool fos,
                        bool rht, uint32_t mask, const int32_t *row_index, int G, const int32_t *row_off,
                        const int32_t *sf_off, const float *scale_src, bool src_is_amax, float *gs_out,
                        bool write_gs, uint8_t *codes, uint8_t *sf, int num_sms, cudaStream_t s);
// amax + NVFP4 16x16 quantize of a contiguous tensor in one cooperative
// kernel.  The first 8 bytes of codes must be zero on entry.  Returns
// non-zero if the launch failed.
int launch_quant_nvfp4_fused(const uint16_t *x, int64_t M, int64_t K, bool rht, uint32_t mask, float *gs_out,
                             uint8_t *codes, uint8_t *sf, unsigned int *err, int num_sms, cudaStream_t s);
// Streaming NVFP4 kernels for contiguous tensors (stream_ok): mode 0 = amax
// only (into *amax_bits, zeroed by the caller; with a counter, also zeroed,
// the last CTA writes s_g to *gs_out), 1 = quantize with s_g from *scale_src
// (an amax when src_is_amax), 2 = amax and quantize in one cooperative
// launch (counter and amax bits in the first 8 bytes of codes, zeroed).
// Returns non-zero if the launch failed.
bool stream_ok(int64_t M, int64_t K, bool block_2d);
int launch_nvfp4_stream(int mode, const uint16_t *x, int64_t M, int64_t K, bool block_2d, bool rht, uint32_t mask,
                        unsigned int *counter, unsigned int *amax_bits, const float *scale_src, bool src_is_amax,
                        float *gs_out, uint8_t *codes, uint8_t *sf, unsigned int *err, int num_sms, cudaStream_t s);
void launch_quant_mxfp8(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, bool colwise, bool sr,
                        uint64_t seed, uint32_t stream_id, uint8_t *codes, uint8_t *sf, int num_sms,
                        cudaStream_t s);
void launch_quant_mxfp8_rowcol(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, bool sr, uint64_t seed,
                               uint32_t stream_r, uint32_t stream_c, uint8_t *codes_r, uint8_t *sf_r,
                               uint8_t *codes_c, uint8_t *sf_c, int num_sms, cudaStream_t s);
void launch_requant_nvfp4_mxfp8(const uint8_t *codes_in, const uint8_t *sf_in, const float *gs, int64_t R, int64_t C,
                                bool sr, uint64_t seed, uint32_t stream_id, uint8_t *codes, uint8_t *sf, int num_sms,
                                cudaStream_t s);
void launch_quant_mxfp4(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, bool sr, uint64_t seed,
                        uint32_t stream_id, uint8_t *codes, uint8_t *sf, int num_sms, cudaStream_t s);
void launch_quant_nvfp4_sr(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, bool block_2d, bool rht,
                           uint32_t mask, const int32_t *row_index, const float *scale_src, bool src_is_amax,
                           float *gs_out, bool write_gs, uint64_t seed, uint32_t stream_id, uint8_t *codes,
                           uint8_t *sf, int num_sms, cudaStream_t s);
void launch_requant_transpose(const uint8_t *codes_row, const uint8_t *sf_row, int64_t M, int64_t K, bool sr,
                              uint64_t seed, uint32_t stream_id, uint8_t *codes_col, uint8_t *sf_col,
                              int num_sms, cudaStream_t s);
void launch_quant_s2f6(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, bool rht, uint32_t mask, int8_t *codes,
                       uint8_t *sf, int num_sms, cudaStream_t s);
void launch_combine_s2f6(const int8_t *codes, const uint8_t *sf, int64_t K, const int32_t *off, const int32_t *rows,
                         const float *weights, int64_t T, uint32_t mask, uint16_t *out, int64_t ldo, int num_sms,
                         cudaStream_t s);
void launch_gather_rows(const void *src, int64_t row_bytes, const int32_t *index, int64_t R, void *dst, int num_sms,
                        cudaStream_t s);
void launch_sf_to_rows(const uint8_t *sf, int64_t rows, int64_t nblk, uint8_t *out, int num_sms, cudaStream_t s);
void launch_sf_from_rows(const uint8_t *in, int64_t rows, int64_t nblk, int G, const int32_t *row_off,
                         const int32_t *sf_off, uint8_t *sf, int num_sms, cudaStream_t s);
void launch_row_absmax(const uint16_t *x, int64_t T, int64_t K, int64_t ldx, bool rht, uint32_t mask, float *rowmax,
                       int num_sms, cudaStream_t s);
void launch_gathered_max(const float *rowmax, const int32_t *row_index, int64_t M, unsigned int *amax_bits,
                         unsigned int *counter, float *gs_out, int num_sms, cudaStream_t s);
void launch_gather_sf(const uint8_t *sf_src, int64_t nblk, const int32_t *row_index, int64_t M, int G,
                      const int32_t *row_off, const int32_t *sf_off, uint8_t *sf, int num_sms, cudaStream_t s);
void launch_rht(const uint16_t *x, uint16_t *y, int64_t M, int64_t K, int64_t ldx, int64_t ldy, uint32_t mask,
                int num_sms, cudaStream_t s);

}  // namespace bsq
