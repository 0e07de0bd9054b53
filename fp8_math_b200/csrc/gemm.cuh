// gemm.cuh -- host interface of the block-scaled GEMM kernels (gemm.cu).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace bsq {

struct GemmArgs {
    int fmt;  // BSQ_NVFP4 / BSQ_MXFP8 / BSQ_MXFP4
    const uint8_t *A, *sfA, *B, *sfB;
    const float *gsA, *gsB;
    int64_t M, N, K;
    void *C;  // may be NULL when the output is quantized (q_codes set)
    int64_t ldc;
    bool out_bf16;
    int G;  // 0: dense; > 0: grouped (MoE experts)
    const int32_t *row_off, *sf_row_off;
    unsigned int *err;
    int num_sms;
    // NVFP4 output (grouped NVFP4 GEMM with the quantizing epilogue): codes,
    // swizzled scales at the groups' SF offsets, the global scale to use,
    // optional amax word, Four Over Six
    uint8_t *q_codes = nullptr, *q_sf = nullptr;
    const float *q_sg = nullptr;
    unsigned int *q_amax = nullptr;
    bool q_fos = false;
};

int launch_gemm(const GemmArgs &g, cudaStream_t s);
void launch_timeout_probe(uint64_t timeout_ns, unsigned int *err, cudaStream_t s);

}  // namespace bsq
