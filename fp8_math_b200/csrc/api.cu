// api.cu -- the C entry points of libbsq (include/bsq.h): argument
// validation, per-device state (SM count, error word), kernel launches.
#include <cstdio>
#include <cstring>
#include <atomic>
#include <cstdlib>
#include <mutex>

#include "common.cuh"
#include "gemm.cuh"
#include "quant.cuh"

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
    bool ready = false;
    int num_sms = 0;
    unsigned int *err = nullptr;  // device error word
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

// Per-device state for the current device; created on first use.
int device_state(DeviceState **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BSQ_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceState &d = g_dev[dev];
    if (!d.ready) {
        if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return BSQ_ERR_CUDA;
        if (cudaMalloc(&d.err, sizeof(unsigned int)) != cudaSuccess) return BSQ_ERR_CUDA;
        if (cudaMemset(d.err, 0, sizeof(unsigned int)) != cudaSuccess) return BSQ_ERR_CUDA;
        d.ready = true;
    }
    *out = &d;
    return BSQ_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int launch_status() { return cudaGetLastError() == cudaSuccess ? BSQ_OK : BSQ_ERR_CUDA; }

// Philox4x32-10 on the host (Salmon et al., SC'11).
void philox_host(uint32_t c[4], uint32_t k0, uint32_t k1) {
    for (int r = 0; r < 10; r++) {
        if (r) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        uint64_t p0 = (uint64_t)0xD2511F53u * c[0];
        uint64_t p1 = (uint64_t)0xCD9E8D57u * c[2];
        uint32_t n0 = (uint32_t)(p1 >> 32) ^ c[1] ^ k0, n1 = (uint32_t)p1;
        uint32_t n2 = (uint32_t)(p0 >> 32) ^ c[3] ^ k1, n3 = (uint32_t)p0;
        c[0] = n0; c[1] = n1; c[2] = n2; c[3] = n3;
    }
}

// Kernel-selection overrides (bsq_debug_kernel_choice): -1 = automatic.
std::atomic<int> g_knob[6] = {{-1}, {-1}, {-1}, {-1}, {-1}, {-1}};

}  // namespace

namespace bsq {
int kernel_choice(int knob) { return g_knob[knob].load(std::memory_order_relaxed); }
}  // namespace bsq

extern "C" {

int bsq_debug_kernel_choice(int knob, int value) {
    switch (knob) {
        case BSQ_KNOB_FUSED_QUANT:
        case BSQ_KNOB_GEMM_PAIR:
        case BSQ_KNOB_STREAM_QUANT:
        case BSQ_KNOB_LAUNCH_OVERLAP:
            if (value < -1 || value > 1) return BSQ_ERR_INVALID;
            break;
        case BSQ_KNOB_GEMM_BN:
            if (value != -1 && value != 128 && value != 256) return BSQ_ERR_INVALID;
            break;
        case BSQ_KNOB_GEMM_SPLITK:
            if (value != -1 && value != 1 && value != 2 && value != 4 && value != 8) return BSQ_ERR_INVALID;
            break;
        default:
            return BSQ_ERR_INVALID;
    }
    g_knob[knob].store(value, std::memory_order_relaxed);
    return BSQ_OK;
}

const char *bsq_status_str(int status) {
    switch (status) {
        case BSQ_OK: return "ok";
        case BSQ_ERR_INVALID: return "invalid argument";
        case BSQ_ERR_ALIGN: return "misaligned pointer or leading dimension";
        case BSQ_ERR_UNSUPPORTED: return "unsupported request";
        case BSQ_ERR_CUDA: return "CUDA error";
        case BSQ_ERR_TIMEOUT: return "device-side wait timed out";
        default: return "unknown status";
    }
}

size_t bsq_sf_bytes(int64_t rows, int64_t nblocks) {
    if (rows < 0 || nblocks < 0) return 0;
    return (size_t)((rows + 127) / 128 * 128) * (size_t)((nblocks + 3) / 4 * 4);
}

uint16_t bsq_rht_sign_mask(uint64_t seed) {
    uint32_t c[4] = {0u, 0u, 0u, 0u};
    philox_host(c, (uint32_t)seed, (uint32_t)(seed >> 32));
    return (uint16_t)(c[0] & 0xFFFFu);
}

static bool stream_enabled(bool block_2d);

int bsq_amax(const void *x, int64_t M, int64_t K, int64_t ldx, int rht_enable, uint16_t mask,
             const int32_t *row_index, float *amax_dev, void *stream) {
    if (!x || !amax_dev || M < 0 || K < 0 || K % 16 || ldx < K) return BSQ_ERR_INVALID;
    if (!aligned16(x) || ldx % 8 || (reinterpret_cast<uintptr_t>(amax_dev) & 3u)) return BSQ_ERR_ALIGN;
    DeviceState *d;
    if (int st = device_state(&d)) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(amax_dev, 0, sizeof(float), s) != cudaSuccess) return BSQ_ERR_CUDA;
    if (M == 0 || K == 0) return BSQ_OK;
    if (!row_index && ldx == K && stream_enabled(false) && bsq::stream_ok(M, K, false)) {
        if (bsq::launch_nvfp4_stream(0, static_cast<const uint16_t *>(x), M, K, false, rht_enable != 0, mask, nullptr,
                                     reinterpret_cast<unsigned int *>(amax_dev), nullptr, false, nullptr, nullptr,
                                     nullptr, d->err, d->num_sms, s) != 0)
            return BSQ_ERR_CUDA;
        return launch_status();
    }
    bsq::launch_amax(static_cast<const uint16_t *>(x), M, K, ldx, rht_enable != 0, mask, row_index,
                     reinterpret_cast<unsigned int *>(amax_dev), nullptr, nullptr, d->num_sms, s);
    return launch_status();
}

// The fused amax + quantize kernel can be switched off
// (bsq_debug_kernel_choice(BSQ_KNOB_FUSED_QUANT, 0)) for tuning and for
// tests of the two-pass path.  It is a cooperative launch with a grid
// barrier; while the stream is being captured into a CUDA graph the two
// passes are launched instead (same bytes), so that a graph holds only
// ordinary kernel nodes.
static bool fused_enabled(cudaStream_t s) {
    cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &st) == cudaSuccess && st != cudaStreamCaptureStatusNone) return false;
    return bsq::kernel_choice(BSQ_KNOB_FUSED_QUANT) != 0;
}
// The bulk-copy streaming kernels for contiguous tensors: by default for
// 16x16 blocks only (on 14336x4096 with the RHT they measure 71.7 us against
// 75.8 for the register-streaming fused kernel; on 8192x4096 with 1x16
// blocks 49.2 us against 45.1 for the two register-streaming passes, and
// 24.6 against 22.6 us for the amax alone).  BSQ_KNOB_STREAM_QUANT forces
// them on (1) or off (0) for every contiguous tensor.
static bool stream_enabled(bool block_2d) {
    const int v = bsq::kernel_choice(BSQ_KNOB_STREAM_QUANT);
    return v < 0 ? block_2d : v != 0;
}

int bsq_quant_nvfp4(const void *x, int64_t M, int64_t K, int64_t ldx, int block_2d, int four_over_six,
                    int rht_enable, uint16_t mask, const int32_t *row_index, int G, const int32_t *row_off,
                    const int32_t *sf_off, const float *amax_in, float *gs, uint8_t *codes, uint8_t *sf,
                    void *stream) {
    if (!x || !gs || !codes || !sf || M < 0 || K < 0 || K % 16 || ldx < K || G < 0) return BSQ_ERR_INVALID;
    if (block_2d && (M % 16 || four_over_six || G > 0)) return BSQ_ERR_INVALID;
    if (G > 0 && (!row_off || !sf_off)) return BSQ_ERR_INVALID;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(sf) || ldx % 8 ||
        (reinterpret_cast<uintptr_t>(gs) & 3u) || (amax_in && (reinterpret_cast<uintptr_t>(amax_in) & 3u)))
        return BSQ_ERR_ALIGN;
    DeviceState *d;
    if (int st = device_state(&d)) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const uint16_t *xx = static_cast<const uint16_t *>(x);
    if (M == 0 || K == 0) {
        // empty tensor: amax 0, s_g = 1
        if (cudaMemsetAsync(gs, 0, sizeof(float), s) != cudaSuccess) return BSQ_ERR_CUDA;
        bsq::launch_finalize_global_scale(gs, s);
        return launch_status();
    }
    const bool streamable = !row_index && G == 0 && ldx == K && !four_over_six && stream_enabled(block_2d != 0) &&
                            bsq::stream_ok(M, K, block_2d != 0);
    if (amax_in == nullptr) {
        // The amax pass uses the first 8 bytes of the caller's code buffer
        // (overwritten by the quantize pass that follows on the same stream)
        // as its scratch: a CTA counter and the amax bits.  Its last CTA
        // writes s_g to *gs, which the quantize pass reads.
        if (cudaMemsetAsync(codes, 0, 8, s) != cudaSuccess) return BSQ_ERR_CUDA;
        if (streamable) {
            unsigned int *scratch = reinterpret_cast<unsigned int *>(codes);
            int rc;
            if (fused_enabled(s)) {
                // amax and quantize in one cooperative launch
                rc = bsq::launch_nvfp4_stream(2, xx, M, K, block_2d != 0, rht_enable != 0, mask, scratch, scratch + 1,
                                              nullptr, false, gs, codes, sf, d->err, d->num_sms, s);
            } else {
                rc = bsq::launch_nvfp4_stream(0, xx, M, K, block_2d != 0, rht_enable != 0, mask, scratch, scratch + 1,
                                              nullptr, false, gs, nullptr, nullptr, d->err, d->num_sms, s);
                if (rc == 0)
                    rc = bsq::launch_nvfp4_stream(1, xx, M, K, block_2d != 0, rht_enable != 0, mask, nullptr, nullptr,
                                                  gs, false, nullptr, codes, sf, d->err, d->num_sms, s);
            }
            return rc ? BSQ_ERR_CUDA : launch_status();
        }
        const int64_t KB = K / 16;
        // (1x16 tensors measure faster with the two-pass path: 37.2 vs 38.3 us
        // on 8192x4096, where the fused kernel's lower occupancy outweighs the
        // L2 reuse; 16x16 tensors gain: 70.9 vs 74.5 us on 14336x4096)
        (void)KB;
        const bool fusable = !row_index && G == 0 && ldx == K && !four_over_six && block_2d && fused_enabled(s);
        if (fusable) {
            // amax and quantize in one cooperative kernel
            if (bsq::launch_quant_nvfp4_fused(xx, M, K, rht_enable != 0, mask, gs, codes, sf, d->err, d->num_sms,
                                              s) != 0)
                return BSQ_ERR_CUDA;
            return launch_status();
        }
        unsigned int *scratch = reinterpret_cast<unsigned int *>(codes);
        bsq::launch_amax(xx, M, K, ldx, rht_enable != 0, mask, row_index, scratch + 1, scratch, gs, d->num_sms, s);
        bsq::launch_quant_nvfp4(xx, M, K, ldx, block_2d != 0, four_over_six != 0, rht_enable != 0, mask, row_index,
                                G, row_off, sf_off, gs, false, gs, false, codes, sf, d->num_sms, s);
    } else if (streamable) {
        // amax given: the quantize pass alone (in place: *gs holds the amax
        // and becomes s_g after the pass)
        const bool in_place = amax_in == gs;
        if (bsq::launch_nvfp4_stream(1, xx, M, K, block_2d != 0, rht_enable != 0, mask, nullptr, nullptr, amax_in, true,
                                     in_place ? nullptr : gs, codes, sf, d->err, d->num_sms, s) != 0)
            return BSQ_ERR_CUDA;
        if (in_place) bsq::launch_finalize_global_scale(gs, s);
    } else if (amax_in == gs) {
        // the caller's amax is in *gs: read it, then replace it by s_g in place
        bsq::launch_quant_nvfp4(xx, M, K, ldx, block_2d != 0, four_over_six != 0, rht_enable != 0, mask, row_index,
                                G, row_off, sf_off, gs, true, gs, false, codes, sf, d->num_sms, s);
        bsq::launch_finalize_global_scale(gs, s);
    } else {
        bsq::launch_quant_nvfp4(xx, M, K, ldx, block_2d != 0, four_over_six != 0, rht_enable != 0, mask, row_index,
                                G, row_off, sf_off, amax_in, true, gs, true, codes, sf, d->num_sms, s);
    }
    return launch_status();
}

// Workspace of bsq_quant_nvfp4_gather: 256 bytes (counter, amax bits), the
// per-row maxima, the source rows' codes and their swizzled scales.
static int64_t gather_ws_rowmax(int64_t) { return 256; }
static int64_t gather_ws_codes(int64_t T) { return (256 + 4 * T + 255) / 256 * 256; }
static int64_t gather_ws_sf(int64_t T, int64_t K) { return gather_ws_codes(T) + (T * (K / 2) + 255) / 256 * 256; }

size_t bsq_quant_nvfp4_gather_workspace(int64_t T, int64_t K) {
    if (T < 0 || K < 0 || K % 16) return 0;
    return (size_t)gather_ws_sf(T, K) + bsq_sf_bytes(T, K / 16);
}

int bsq_quant_nvfp4_gather(const void *x, int64_t T, int64_t K, int64_t ldx, const int32_t *row_index, int64_t M,
                           int four_over_six, int rht_enable, uint16_t mask, int G, const int32_t *row_off,
                           const int32_t *sf_off, const float *amax_in, float *gs, uint8_t *codes, uint8_t *sf,
                           void *workspace, size_t workspace_bytes, void *stream) {
    if (!x || !row_index || !gs || !codes || !sf || !workspace || T < 0 || M < 0 || K < 0 || K % 64 || ldx < K ||
        G < 0 || (G > 0 && (!row_off || !sf_off)))
        return BSQ_ERR_INVALID;
    if (workspace_bytes < bsq_quant_nvfp4_gather_workspace(T, K)) return BSQ_ERR_INVALID;
    if (G > 1024) return BSQ_ERR_UNSUPPORTED;  // the scale mover keeps the offsets in shared memory
    if (!aligned16(x) || !aligned16(codes) || !aligned16(sf) || ldx % 8 || (reinterpret_cast<uintptr_t>(gs) & 3u) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) || (amax_in && (reinterpret_cast<uintptr_t>(amax_in) & 3u)))
        return BSQ_ERR_ALIGN;
    DeviceState *d;
    if (int st = device_state(&d)) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const uint16_t *xx = static_cast<const uint16_t *>(x);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    unsigned int *scratch = reinterpret_cast<unsigned int *>(ws);
    float *rowmax = reinterpret_cast<float *>(ws + gather_ws_rowmax(T));
    uint8_t *codes_src = ws + gather_ws_codes(T);
    uint8_t *sf_src = ws + gather_ws_sf(T, K);
    if (M == 0 || K == 0 || T == 0) {
        if (cudaMemsetAsync(gs, 0, sizeof(float), s) != cudaSuccess) return BSQ_ERR_CUDA;
        bsq::launch_finalize_global_scale(gs, s);
        return launch_status();
    }
    if (amax_in == nullptr) {
        if (cudaMemsetAsync(scratch, 0, 8, s) != cudaSuccess) return BSQ_ERR_CUDA;
        bsq::launch_row_absmax(xx, T, K, ldx, rht_enable != 0, mask, rowmax, d->num_sms, s);
        bsq::launch_gathered_max(rowmax, row_index, M, scratch + 1, scratch, gs, d->num_sms, s);
        bsq::launch_quant_nvfp4(xx, T, K, ldx, false, four_over_six != 0, rht_enable != 0, mask, nullptr, 0, nullptr,
                                nullptr, gs, false, gs, false, codes_src, sf_src, d->num_sms, s);
    } else if (amax_in == gs) {
        bsq::launch_quant_nvfp4(xx, T, K, ldx, false, four_over_six != 0, rht_enable != 0, mask, nullptr, 0, nullptr,
                                nullptr, gs, true, gs, false, codes_src, sf_src, d->num_sms, s);
        bsq::launch_finalize_global_scale(gs, s);
    } else {
        bsq::launch_quant_nvfp4(xx, T, K, ldx, false, four_over_six != 0, rht_enable != 0, mask, nullptr, 0, nullptr,
                                nullptr, amax_in, true, gs, true, codes_src, sf_src, d->num_sms, s);
    }
    bsq::launch_gather_rows(codes_src, K / 2, row_index, M, codes, d->num_sms, s);
    bsq::launch_gather_sf(sf_src, K / 16, row_index, M, G, row_off, sf_off, sf, d->num_sms, s);
    return launch_status();
}

int bsq_quant_nvfp4_sr(const void *x, int64_t M, int64_t K, int64_t ldx, int block_2d, int rht_enable, uint16_t mask,
                       const int32_t *row_index, const float *amax_in, float *gs, uint64_t seed, uint32_t stream_id,
                       uint8_t *codes, uint8_t *sf, void *stream) {
    if (!x || !gs || !codes || !sf || M < 0 || K < 0 || K % 16 || ldx < K) return BSQ_ERR_INVALID;
    if (block_2d && (M % 16 || row_index)) return BSQ_ERR_INVALID;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(sf) || ldx % 8 ||
        (reinterpret_cast<uintptr_t>(gs) & 3u) || (amax_in && (reinterpret_cast<uintptr_t>(amax_in) & 3u)))
        return BSQ_ERR_ALIGN;
    DeviceState *d;
    if (int st = device_state(&d)) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const uint16_t *xx = static_cast<const uint16_t *>(x);
    if (M == 0 || K == 0) {
        if (cudaMemsetAsync(gs, 0, sizeof(float), s) != cudaSuccess) return BSQ_ERR_CUDA;
        bsq::launch_finalize_global_scale(gs, s);
        return launch_status();
    }
    if (amax_in == nullptr) {
        // the amax pass's scratch is the first 8 bytes of codes, as in bsq_quant_nvfp4
        if (cudaMemsetAsync(codes, 0, 8, s) != cudaSuccess) return BSQ_ERR_CUDA;
        unsigned int *scratch = reinterpret_cast<unsigned int *>(codes);
        bsq::launch_amax(xx, M, K, ldx, rht_enable != 0, mask, row_index, scratch + 1, scratch, gs, d->num_sms, s);
        bsq::launch_quant_nvfp4_sr(xx, M, K, ldx, block_2d != 0, rht_enable != 0, mask, row_index, gs, false, gs,
                                   false, seed, stream_id, codes, sf, d->num_sms, s);
    } else if (amax_in == gs) {
        bsq::launch_quant_nvfp4_sr(xx, M, K, ldx, block_2d != 0, rht_enable != 0, mask, row_index, gs, true, gs,
                                   false, seed, stream_id, codes, sf, d->num_sms, s);
        bsq::launch_finalize_global_scale(gs, s);
    } else {
        bsq::launch_quant_nvfp4_sr(xx, M, K, ldx, block_2d != 0, rht_enable != 0, mask, row_index, amax_in, true, gs,
                                   true, seed, stream_id, codes, sf, d->num_sms, s);
    }
    return launch_status();
}

int bsq_quant_mxfp8(const void *x, int64_t M, int64_t K, int64_t ldx, int colwise, int rounding, uint64_t seed,
                    uint32_t stream_id, uint8_t *codes, uint8_t *sf, void *stream) {
    if (!x || !codes || !sf || M < 0 || K < 0 || ldx < K || (rounding != BSQ_RNE && rounding != BSQ_SR))
        return BSQ_ERR_INVALID;
    if (colwise ? (M % 32 || K % 8) : (K % 32)) return BSQ_ERR_INVALID;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(sf) || ldx % 8) return BSQ_ERR_ALIGN;
    if (colwise && M % 16) return BSQ_ERR_ALIGN;
    if (colwise && (M >> 5) * ((K + 63) >> 6) >= (int64_t(1) << 31)) return BSQ_ERR_UNSUPPORTED;
    DeviceState *d;
    if (int st = device_state(&d)) return st;
    if (M == 0 || K == 0) return BSQ_OK;
    bsq::launch_quant_mxfp8(static_cast<const uint16_t *>(x), M, K, ldx, colwise != 0, rounding == BSQ_SR, seed,
                            stream_id, codes, sf, d->num_sms, static_cast<cudaStream_t>(stream));
    return launch_status();
}

int bsq_quant_mxfp8_rowcol(const void *x, int64_t M, int64_t K, int64_t ldx, int rounding, uint64_t seed,
                           uint32_t stream_id_row, uint32_t stream_id_col, uint8_t *codes_row, uint8_t *sf_row,
                           uint8_t *codes_col, uint8_t *sf_col, void *stream) {
    if (!x || !codes_row || !sf_row || !codes_col || !sf_col || M < 0 || K < 0 || ldx < K || M % 32 || K % 32 ||
        (rounding != BSQ_RNE && rounding != BSQ_SR))
        return BSQ_ERR_INVALID;
    if (!aligned16(x) || !aligned16(codes_row) || !aligned16(sf_row) || !aligned16(codes_col) || !aligned16(sf_col) ||
        ldx % 8)
        return BSQ_ERR_ALIGN;
    if ((M >> 5) * ((K + 63) >> 6) >= (int64_t(1) << 31)) return BSQ_ERR_UNSUPPORTED;
    DeviceState *d;
    if (int st = device_state(&d)) return st;
    if (M == 0 || K == 0) return BSQ_OK;
    bsq::launch_quant_mxfp8_rowcol(static_cast<const uint16_t *>(x), M, K, ldx, rounding == BSQ_SR, seed,
                                   stream_id_row, stream_id_col, codes_row, sf_row, codes_col, sf_col, d->num_sms,
                                   static_cast<cudaStream_t>(stream));
    return launch_status();
}

int bsq_requant_nvfp4_mxfp8(const uint8_t *codes, const uint8_t *sf, const float *gs_dev, int64_t R, int64_t C,
                            int rounding, uint64_t seed, uint32_t stream_id, uint8_t *codes_col, uint8_t *sf_col,
                            void *stream) {
    if (!codes || !sf || !gs_dev || !codes_col || !sf_col || R < 0 || C < 0 || R % 32 || C % 16 ||
        (rounding != BSQ_RNE && rounding != BSQ_SR))
        return BSQ_ERR_INVALID;
    if (!aligned16(codes) || !aligned16(sf) || !aligned16(codes_col) || !aligned16(sf_col) ||
        (reinterpret_cast<uintptr_t>(gs_dev) & 3u))
        return BSQ_ERR_ALIGN;
    if ((R >> 5) * ((C + 63) >> 6) >= (int64_t(1) << 31)) return BSQ_ERR_UNSUPPORTED;
    DeviceState *d;
    if (int st = device_state(&d)) return st;
    if (R == 0 || C == 0) return BSQ_OK;
    bsq::launch_requant_nvfp4_mxfp8(codes, sf, gs_dev, R, C, rounding == BSQ_SR, seed, stream_id, codes_col, sf_col,
                                    d->num_sms, static_cast<cudaStream_t>(stream));
    return launch_status();
}

int bsq_quant_mxfp4(const void *x, int64_t M, int64_t K, int64_t ldx, int rounding, uint64_t seed,
                    uint32_t stream_id, uint8_t *codes, uint8_t *sf, void *stream) {
    if (!x || !codes || !sf || M < 0 || K < 0 || ldx < K || K % 32 || (rounding != BSQ_RNE && rounding != BSQ_SR))
        return BSQ_ERR_INVALID;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(sf) || ldx % 8) return BSQ_ERR_ALIGN;
    DeviceState *d;
    if (int st = device_state(&d)) return st;
    if (M == 0 || K == 0) return BSQ_OK;
    bsq::launch_quant_mxfp4(static_cast<const uint16_t *>(x), M, K, ldx, rounding == BSQ_SR, seed, stream_id, codes,
                            sf, d->num_sms, static_cast<cudaStream_t>(stream));
    return launch_status();
}

int bsq_quant_s2f6(const void *x, int64_t M, int64_t K, int64_t ldx, int rht_enable, uint16_t mask, int8_t *codes,
                   uint8_t *sf, void *stream) {
    if (!x || !codes || !sf || M < 0 || K < 0 || K % 32 || ldx < K) return BSQ_ERR_INVALID;
    if (!aligned16(x) || !aligned16(codes) || ldx % 8) return BSQ_ERR_ALIGN;
    DeviceState *d;
    if (int st = device_state(&d)) return st;
    if (M == 0 || K == 0) return BSQ_OK;
    bsq::launch_quant_s2f6(static_cast<const uint16_t *>(x), M, K, ldx, rht_enable != 0, mask, codes, sf, d->num_sms,
                           static_cast<cudaStream_t>(stream));
    return launch_status();
}

int bsq_combine_s2f6(const int8_t *codes, const uint8_t *sf, int64_t K, const int32_t *token_offsets,
                     const int32_t *rows, const float *weights, int64_t T, uint16_t mask, void *out_bf16,
                     int64_t ldo, void *stream) {
    if (!codes || !sf || !token_offsets || !out_bf16 || K < 0 || K % 32 || T < 0 || ldo < K) return BSQ_ERR_INVALID;
    if (!aligned16(codes) || !aligned16(out_bf16) || ldo % 8 || (reinterpret_cast<uintptr_t>(token_offsets) & 3u) ||
        (reinterpret_cast<uintptr_t>(rows) & 3u) || (reinterpret_cast<uintptr_t>(weights) & 3u))
        return BSQ_ERR_ALIGN;
    DeviceState *d;
    if (int st = device_state(&d)) return st;
    if (T == 0 || K == 0) return BSQ_OK;
    if (!rows || !weights) return BSQ_ERR_INVALID;
    bsq::launch_combine_s2f6(codes, sf, K, token_offsets, rows, weights, T, mask, static_cast<uint16_t *>(out_bf16), ldo,
                             d->num_sms, static_cast<cudaStream_t>(stream));
    return launch_status();
}

int bsq_gather_rows(const void *src, int64_t row_bytes, const int32_t *index, int64_t R, void *dst, void *stream) {
    if (!src || !dst || R < 0 || row_bytes < 0 || row_bytes % 16 || (R > 0 && !index)) return BSQ_ERR_INVALID;
    if (!aligned16(src) || !aligned16(dst) || (reinterpret_cast<uintptr_t>(index) & 3u)) return BSQ_ERR_ALIGN;
    DeviceState *d;
    if (int st = device_state(&d)) return st;
    if (R == 0 || row_bytes == 0) return BSQ_OK;
    bsq::launch_gather_rows(src, row_bytes, index, R, dst, d->num_sms, static_cast<cudaStream_t>(stream));
    return launch_status();
}

int bsq_sf_to_rows(const uint8_t *sf, int64_t rows, int64_t nblk, uint8_t *out, void *stream) {
    if (!sf || !out || rows < 0 || nblk < 0) return BSQ_ERR_INVALID;
    if (rows * nblk >= (int64_t(1) << 31)) return BSQ_ERR_UNSUPPORTED;  // 32-bit indexing
    DeviceState *d;
    if (int st = device_state(&d)) return st;
    if (rows == 0 || nblk == 0) return BSQ_OK;
    bsq::launch_sf_to_rows(sf, rows, nblk, out, d->num_sms, static_cast<cudaStream_t>(stream));
    return launch_status();
}

int bsq_sf_from_rows(const uint8_t *in, int64_t rows, int64_t nblk, int G, const int32_t *row_off,
                     const int32_t *sf_row_off, uint8_t *sf, void *stream) {
    if (!in || !sf || rows < 0 || nblk < 0 || G < 0 || (G > 0 && (!row_off || !sf_row_off))) return BSQ_ERR_INVALID;
    if (rows * nblk >= (int64_t(1) << 31)) return BSQ_ERR_UNSUPPORTED;  // 32-bit indexing
    DeviceState *d;
    if (int st = device_state(&d)) return st;
    if (rows == 0 || nblk == 0) return BSQ_OK;
    bsq::launch_sf_from_rows(in, rows, nblk, G, row_off, sf_row_off, sf, d->num_sms, static_cast<cudaStream_t>(stream));
    return launch_status();
}

int bsq_rht(const void *x, void *y, int64_t M, int64_t K, int64_t ldx, int64_t ldy, uint16_t mask, void *stream) {
    if (!x || !y || M < 0 || K < 0 || K % 16 || ldx < K || ldy < K) return BSQ_ERR_INVALID;
    if (!aligned16(x) || !aligned16(y) || ldx % 8 || ldy % 8) return BSQ_ERR_ALIGN;
    if (x == y && ldx != ldy) return BSQ_ERR_INVALID;
    DeviceState *d;
    if (int st = device_state(&d)) return st;
    if (M == 0 || K == 0) return BSQ_OK;
    bsq::launch_rht(static_cast<const uint16_t *>(x), static_cast<uint16_t *>(y), M, K, ldx, ldy, mask, d->num_sms,
                    static_cast<cudaStream_t>(stream));
    return launch_status();
}

int bsq_requant_transpose(const uint8_t *codes_row, const uint8_t *sf_row, int64_t M, int64_t K, int rounding,
                          uint64_t seed, uint32_t stream_id, uint8_t *codes_col, uint8_t *sf_col, void *stream) {
    if (!codes_row || !sf_row || !codes_col || !sf_col || M < 0 || K < 0 || M % 32 || K % 32 ||
        (rounding != BSQ_RNE && rounding != BSQ_SR))
        return BSQ_ERR_INVALID;
    if (!aligned16(codes_row) || !aligned16(sf_row) || !aligned16(codes_col) || !aligned16(sf_col))
        return BSQ_ERR_ALIGN;
    if ((M >> 5) * ((K + 63) >> 6) >= (int64_t(1) << 31)) return BSQ_ERR_UNSUPPORTED;
    DeviceState *d;
    if (int st = device_state(&d)) return st;
    if (M == 0 || K == 0) return BSQ_OK;
    bsq::launch_requant_transpose(codes_row, sf_row, M, K, rounding == BSQ_SR, seed, stream_id, codes_col, sf_col,
                                  d->num_sms, static_cast<cudaStream_t>(stream));
    return launch_status();
}

int bsq_gemm_blockscaled(int fmt, const uint8_t *A, const uint8_t *sfA, const float *gsA, const uint8_t *B,
                         const uint8_t *sfB, const float *gsB, int64_t M, int64_t N, int64_t K, void *C, int64_t ldc,
                         int out_type, void *stream) {
    if ((fmt != BSQ_NVFP4 && fmt != BSQ_MXFP8 && fmt != BSQ_MXFP4) || (out_type != BSQ_OUT_F32 && out_type != BSQ_OUT_BF16))
        return BSQ_ERR_INVALID;
    if (!A || !sfA || !B || !sfB || !C || M < 1 || N < 1 || K < 128 || K % 128 || ldc < N) return BSQ_ERR_INVALID;
    if (M > (1LL << 31) - 1 || N > (1LL << 31) - 1 || K > (1LL << 31) - 1) return BSQ_ERR_UNSUPPORTED;
    if (!aligned16(A) || !aligned16(B) || !aligned16(sfA) || !aligned16(sfB) || !aligned16(C) ||
        (ldc * (out_type == BSQ_OUT_F32 ? 4 : 2)) % 16)
        return BSQ_ERR_ALIGN;
    DeviceState *d;
    if (int st = device_state(&d)) return st;
    bsq::GemmArgs g{};
    g.fmt = fmt;
    g.A = A; g.sfA = sfA; g.B = B; g.sfB = sfB; g.gsA = gsA; g.gsB = gsB;
    g.M = M; g.N = N; g.K = K; g.C = C; g.ldc = ldc; g.out_bf16 = out_type == BSQ_OUT_BF16;
    g.G = 0;
    g.err = d->err;
    g.num_sms = d->num_sms;
    return bsq::launch_gemm(g, static_cast<cudaStream_t>(stream));
}

int bsq_grouped_gemm(int fmt, int G, const int32_t *row_off, const int32_t *sf_row_off, int64_t M_total,
                     const uint8_t *A, const uint8_t *sfA, const float *gsA, const uint8_t *B, const uint8_t *sfB,
                     const float *gsB, int64_t N, int64_t K, void *C, int64_t ldc, int out_type, void *stream) {
    if ((fmt != BSQ_NVFP4 && fmt != BSQ_MXFP8 && fmt != BSQ_MXFP4) || (out_type != BSQ_OUT_F32 && out_type != BSQ_OUT_BF16))
        return BSQ_ERR_INVALID;
    if (G < 1 || !row_off || !sf_row_off || !A || !sfA || !B || !sfB || !C || M_total < 0 || N < 1 || K < 128 ||
        K % 128 || ldc < N)
        return BSQ_ERR_INVALID;
    if (G > 1024) return BSQ_ERR_UNSUPPORTED;
    if (!aligned16(A) || !aligned16(B) || !aligned16(sfA) || !aligned16(sfB) || !aligned16(C) ||
        (ldc * (out_type == BSQ_OUT_F32 ? 4 : 2)) % 16)
        return BSQ_ERR_ALIGN;
    DeviceState *d;
    if (int st = device_state(&d)) return st;
    if (M_total == 0) return BSQ_OK;
    bsq::GemmArgs g{};
    g.fmt = fmt;
    g.A = A; g.sfA = sfA; g.B = B; g.sfB = sfB; g.gsA = gsA; g.gsB = gsB;
    g.M = M_total; g.N = N; g.K = K; g.C = C; g.ldc = ldc; g.out_bf16 = out_type == BSQ_OUT_BF16;
    g.G = G; g.row_off = row_off; g.sf_row_off = sf_row_off;
    g.err = d->err;
    g.num_sms = d->num_sms;
    return bsq::launch_gemm(g, static_cast<cudaStream_t>(stream));
}

int bsq_grouped_gemm_nvfp4_out(int fmt, int G, const int32_t *row_off, const int32_t *sf_row_off, int64_t M_total,
                               const uint8_t *A, const uint8_t *sfA, const float *gsA, const uint8_t *B,
                               const uint8_t *sfB, const float *gsB, int64_t N, int64_t K, const float *out_gs,
                               int four_over_six, uint8_t *out_codes, uint8_t *out_sf, float *out_amax, void *C,
                               int64_t ldc, void *stream) {
    if (fmt != BSQ_NVFP4) return fmt == BSQ_MXFP8 || fmt == BSQ_MXFP4 ? BSQ_ERR_UNSUPPORTED : BSQ_ERR_INVALID;
    if (G < 1 || !row_off || !sf_row_off || !A || !sfA || !B || !sfB || !out_gs || !out_codes || !out_sf ||
        M_total < 0 || N < 128 || N % 64 || K < 256 || K % 256 || (C && ldc < N))
        return BSQ_ERR_INVALID;
    if (G > 1024) return BSQ_ERR_UNSUPPORTED;
    if (!aligned16(A) || !aligned16(B) || !aligned16(sfA) || !aligned16(sfB) || !aligned16(out_codes) ||
        !aligned16(out_sf) || (reinterpret_cast<uintptr_t>(out_gs) & 3u) ||
        (out_amax && (reinterpret_cast<uintptr_t>(out_amax) & 3u)) || (C && (!aligned16(C) || (ldc * 2) % 16)))
        return BSQ_ERR_ALIGN;
    DeviceState *d;
    if (int st = device_state(&d)) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (out_amax && cudaMemsetAsync(out_amax, 0, sizeof(float), s) != cudaSuccess) return BSQ_ERR_CUDA;
    if (M_total == 0) return BSQ_OK;
    bsq::GemmArgs g{};
    g.fmt = fmt;
    g.A = A; g.sfA = sfA; g.B = B; g.sfB = sfB; g.gsA = gsA; g.gsB = gsB;
    g.M = M_total; g.N = N; g.K = K; g.C = C; g.ldc = C ? ldc : N; g.out_bf16 = true;
    g.G = G; g.row_off = row_off; g.sf_row_off = sf_row_off;
    g.err = d->err;
    g.num_sms = d->num_sms;
    g.q_codes = out_codes; g.q_sf = out_sf; g.q_sg = out_gs;
    g.q_amax = reinterpret_cast<unsigned int *>(out_amax); g.q_fos = four_over_six != 0;
    return bsq::launch_gemm(g, s);
}

int bsq_check(void *stream) {
    DeviceState *d;
    if (int st = device_state(&d)) return st;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return BSQ_ERR_CUDA;
    unsigned int w = 0;
    if (cudaMemcpy(&w, d->err, sizeof w, cudaMemcpyDeviceToHost) != cudaSuccess) return BSQ_ERR_CUDA;
    if (w) {
        if (cudaMemset(d->err, 0, sizeof w) != cudaSuccess) return BSQ_ERR_CUDA;
        return BSQ_ERR_TIMEOUT;
    }
    return BSQ_OK;
}

// ------------------------------------------------------------ no-alloc global scale
// bsq_global_scale_noalloc keeps its scratch in a file-scope device array
// instead of any allocation.  Host code may not use the array's name as a
// device address: the address is looked up with cudaGetSymbolAddress once
// per device, with that device current, and passed to the kernel.
}  // extern "C"

namespace {
constexpr int64_t kNoAllocScratchWords = 4096;  // 16 KiB: a CTA counter + 4095 per-CTA maxima
__device__ __align__(256) unsigned int g_noalloc_scratch[kNoAllocScratchWords];
std::mutex g_noalloc_mu;
unsigned int *g_noalloc_ptr[kMaxDevices];
}  // namespace

extern "C" {

int bsq_global_scale_noalloc(const void *x, int64_t M, int64_t K, int64_t ldx, int rht_enable, uint16_t mask,
                             float *gs_dev, void *stream) {
    if (!x || !gs_dev || M < 0 || K < 0 || K % 16 || ldx < K) return BSQ_ERR_INVALID;
    if (!aligned16(x) || ldx % 8 || (reinterpret_cast<uintptr_t>(gs_dev) & 3u)) return BSQ_ERR_ALIGN;
    // one partial maximum per CTA of kPartialBlocks blocks, plus the counter
    if (M > (int64_t(1) << 40) || K > (int64_t(1) << 40)) return BSQ_ERR_UNSUPPORTED;
    const int64_t ctas = (M * (K / 16) + bsq::kPartialBlocks - 1) / bsq::kPartialBlocks;
    if (1 + ctas > kNoAllocScratchWords) return BSQ_ERR_UNSUPPORTED;  // the array is all there is
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BSQ_ERR_CUDA;
    unsigned int *scratch;
    {
        std::lock_guard<std::mutex> lk(g_noalloc_mu);
        if (!g_noalloc_ptr[dev]) {
            void *ptr = nullptr;
            if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return BSQ_ERR_CUDA;
            g_noalloc_ptr[dev] = static_cast<unsigned int *>(ptr);
        }
        scratch = g_noalloc_ptr[dev];
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (ctas == 0) {
        if (cudaMemsetAsync(gs_dev, 0, sizeof(float), s) != cudaSuccess) return BSQ_ERR_CUDA;
        bsq::launch_finalize_global_scale(gs_dev, s);  // amax 0 gives s_g = 1
        return launch_status();
    }
    // the counter must start at zero; the partials are written before they are read
    if (cudaMemsetAsync(scratch, 0, sizeof(unsigned int), s) != cudaSuccess) return BSQ_ERR_CUDA;
    bsq::launch_amax_partials(static_cast<const uint16_t *>(x), M, K, ldx, rht_enable != 0, mask, scratch, gs_dev, s);
    return launch_status();
}

int bsq_debug_timeout_probe(uint64_t timeout_ns, void *stream) {
    if (timeout_ns == 0 || timeout_ns > 10000000000ull) return BSQ_ERR_INVALID;
    DeviceState *d;
    if (int st = device_state(&d)) return st;
    bsq::launch_timeout_probe(timeout_ns, d->err, static_cast<cudaStream_t>(stream));
    return launch_status();
}

}  // extern "C"
