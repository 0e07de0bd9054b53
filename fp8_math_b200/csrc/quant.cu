// quant.cu -- memory-bound codec kernels of libbsq (sm_100a):
//   tensor amax (optionally of the RHT output), NVFP4 quantize (1x16 with
//   optional Four Over Six, row gather and expert groups; 16x16 tiles),
//   MXFP8 quantize (row-wise, column-wise; RNE or Philox SR), dequantize ->
//   transpose -> requantize, and the standalone 16-point RHT.
// All of them stream bf16/fp8 from HBM with 16-byte vector loads, reduce the
// block amax with warp shuffles, and write packed codes plus scale factors
// directly in the swizzled layout the block-scaled MMA reads.
#include "common.cuh"
#include "quant.cuh"

namespace bsq {

// ===================================================================== amax
// Work mapping shared by the row-oriented kernels: a CTA of 256 threads
// covers (256 >> lpr_shift) rows per step; lanes_per_row = 1 << lpr_shift
// threads walk a row's units, so no index needs an integer division.
struct RowMap {
    int lpr_shift;  // log2(lanes per row)
};

static int lpr_shift_for(int64_t units_per_row) {
    int sh = 0;
    while (sh < 8 && (int64_t(1) << sh) < units_per_row) sh++;
    return sh;
}

template <bool RHT, bool GATHER>
__global__ void __launch_bounds__(256) amax_kernel(const uint16_t *__restrict__ x, int64_t M, int64_t K,
                                                   int64_t ldx, uint32_t mask,
                                                   const int32_t *__restrict__ row_index,
                                                   unsigned int *amax_bits, RowMap map) {
    const int64_t KB = K >> 4;
    const int lpr = 1 << map.lpr_shift;
    const int rpi = 256 >> map.lpr_shift;
    const int sub = threadIdx.x >> map.lpr_shift, lk = threadIdx.x & (lpr - 1);
    uint32_t sw[8];
    rht_sign_words(mask, sw);
    float m = 0.0f;
    for (int64_t r0 = (int64_t)blockIdx.x * rpi; r0 < M; r0 += (int64_t)gridDim.x * rpi) {
        const int64_t row = r0 + sub;
        if (row >= M) continue;
        const int64_t src = GATHER ? (int64_t)__ldg(row_index + row) : row;
        const uint16_t *rp = x + src * ldx;
        for (int64_t kb = lk; kb < KB; kb += lpr) {
            f32x2 P[8];
            if (RHT) load_rht16(rp + kb * 16, sw, P);
            else load16_pairs(rp + kb * 16, P);
            m = fmaxf(m, pairs_absmax(P));
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    __shared__ float red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float b = red[0];
        for (int i = 1; i < (int)(blockDim.x >> 5); i++) b = fmaxf(b, red[i]);
        // non-negative floats order like their bit patterns
        atomicMax(amax_bits, __float_as_uint(b));
    }
}

// s_g = amax / (6 * 448); amax == 0 gives 1.
BSQ_DEV float global_scale_of(float amax) { return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 2688.0f); }

__global__ void finalize_global_scale_kernel(float *gs) { *gs = global_scale_of(*gs); }

// ===================================================================== NVFP4
// One NVFP4 candidate for a 1x16 row segment: scale code, den, packed codes.
struct NvCand {
    uint32_t sb;
    float den;
    uint2 codes;
};

BSQ_DEV NvCand nv_candidate(const f32x2 P[8], float bamax, float divisor, float s_g) {
    NvCand c;
    float t = __fdiv_rn(__fdiv_rn(bamax, divisor), s_g);
    c.sb = e4m3_rne(t);
    float sbv = e4m3_to_f32(c.sb);
    if (sbv == 0.0f) {
        c.den = 0.0f;
        c.codes = make_uint2(0u, 0u);
        return c;
    }
    c.den = __fmul_rn(sbv, s_g);
    const float r = __frcp_rn(c.den);
    const f32x2 R = f2_pack(r, r);
    float q[16];
#pragma unroll
    for (int k = 0; k < 8; k++) f2_unpack(f2_mul(P[k], R), q[2 * k], q[2 * k + 1]);
    c.codes.x = cvt_e2m1x8(q);
    c.codes.y = cvt_e2m1x8(q + 8);
    return c;
}

// Squared error of a candidate, summed pairwise (0+1),(2+3),... four levels.
BSQ_DEV float nv_block_err(const f32x2 P[8], const NvCand &c) {
    float v[16];
#pragma unroll
    for (int k = 0; k < 8; k++) f2_unpack(P[k], v[2 * k], v[2 * k + 1]);
    float e[16];
#pragma unroll
    for (int i = 0; i < 16; i++) {
        uint32_t w = (i < 8) ? c.codes.x : c.codes.y;
        uint32_t code = (w >> (4 * (i & 7))) & 15u;
        float deq = __fmul_rn(e2m1_to_f32(code), c.den);
        float d = __fsub_rn(v[i], deq);
        e[i] = __fmul_rn(d, d);
    }
#pragma unroll
    for (int w = 16; w > 1; w >>= 1)
#pragma unroll
        for (int i = 0; i < w / 2; i++) e[i] = __fadd_rn(e[2 * i], e[2 * i + 1]);
    return e[0];
}

// Row -> scale-factor row under expert groups (binary search of offsets).
BSQ_DEV int64_t grouped_sf_row(int64_t row, int G, const int32_t *__restrict__ off,
                               const int32_t *__restrict__ sfoff) {
    int lo = 0, hi = G;  // off[lo] <= row < off[hi]
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if ((int64_t)__ldg(off + mid) <= row) lo = mid; else hi = mid;
    }
    return row - (int64_t)__ldg(off + lo) + (int64_t)__ldg(sfoff + lo);
}

// Writes the scale byte of a unit: packs 4 consecutive blocks into one word
// when the row's block count is a multiple of 4 (lanes 4j..4j+3 hold blocks
// 4i..4i+3 of one row), else stores the byte.
BSQ_DEV void store_sf(uint8_t *sf, bool valid, uint32_t sb, int64_t sf_row, int64_t kb, int64_t KB, bool pack4) {
    if (pack4) {
        uint32_t b1 = __shfl_down_sync(0xFFFFFFFFu, sb, 1);
        uint32_t b2 = __shfl_down_sync(0xFFFFFFFFu, sb, 2);
        uint32_t b3 = __shfl_down_sync(0xFFFFFFFFu, sb, 3);
        if (valid && (threadIdx.x & 3) == 0) {
            uint32_t w = (sb & 0xFFu) | ((b1 & 0xFFu) << 8) | ((b2 & 0xFFu) << 16) | ((b3 & 0xFFu) << 24);
            *reinterpret_cast<uint32_t *>(sf + sf_word_offset(sf_row, kb >> 2, KB)) = w;
        }
    } else if (valid) {
        sf[sf_offset(sf_row, kb, KB)] = (uint8_t)sb;
    }
}

// 1x16 blocks: one thread per block of 16 (two 16-byte loads, one 8-byte
// code store).  Loops are warp-uniform so that shuffles see all lanes.
template <bool RHT, bool FOS, bool GATHER, bool GROUPED>
__global__ void __launch_bounds__(256) quant_nvfp4_1d_kernel(
    const uint16_t *__restrict__ x, int64_t M, int64_t K, int64_t ldx, uint32_t mask,
    const int32_t *__restrict__ row_index, int G, const int32_t *__restrict__ row_off,
    const int32_t *__restrict__ sf_off, const float *amax_ptr, float *gs_out, int write_gs,
    uint8_t *__restrict__ codes, uint8_t *__restrict__ sf, RowMap map) {
    const int64_t KB = K >> 4;
    const bool pack4 = (KB & 3) == 0;
    const float s_g = global_scale_of(*amax_ptr);
    if (write_gs && blockIdx.x == 0 && threadIdx.x == 0) *gs_out = s_g;
    uint32_t sw[8];
    rht_sign_words(mask, sw);
    const int lpr = 1 << map.lpr_shift;
    const int rpi = 256 >> map.lpr_shift;
    const int sub = threadIdx.x >> map.lpr_shift, lk = threadIdx.x & (lpr - 1);
    for (int64_t r0 = (int64_t)blockIdx.x * rpi; r0 < M; r0 += (int64_t)gridDim.x * rpi) {
        const int64_t row = r0 + sub;
        const bool row_ok = row < M;
        const int64_t rr = row_ok ? row : M - 1;
        const int64_t src = GATHER ? (int64_t)__ldg(row_index + rr) : rr;
        const uint16_t *rp = x + src * ldx;
        const int64_t sf_row = GROUPED ? grouped_sf_row(rr, G, row_off, sf_off) : rr;
        for (int64_t kb0 = 0; kb0 < KB; kb0 += lpr) {
            const int64_t kb = kb0 + lk;
            const bool valid = row_ok && kb < KB;
            const int64_t kk = kb < KB ? kb : KB - 1;
            f32x2 P[8];
            if (RHT) load_rht16(rp + kk * 16, sw, P);
            else load16_pairs(rp + kk * 16, P);
            const float bamax = pairs_absmax(P);
            NvCand c = nv_candidate(P, bamax, 6.0f, s_g);
            if (FOS) {
                NvCand c4 = nv_candidate(P, bamax, 4.0f, s_g);
                if (nv_block_err(P, c4) < nv_block_err(P, c)) c = c4;
            }
            if (valid) *reinterpret_cast<uint2 *>(codes + rr * (K >> 1) + kb * 8) = c.codes;
            store_sf(sf, valid, c.sb, sf_row, kb, KB, pack4);
        }
    }
}

// 16x16 tiles: a CTA of 16 warps covers 16 rows x 32 blocks; warp w owns row
// w of the tile, lane j block j.  The tile amax goes through shared memory.
template <bool RHT>
__global__ void __launch_bounds__(512) quant_nvfp4_2d_kernel(
    const uint16_t *__restrict__ x, int64_t M, int64_t K, int64_t ldx, uint32_t mask,
    const float *amax_ptr, float *gs_out, int write_gs, uint8_t *__restrict__ codes, uint8_t *__restrict__ sf) {
    __shared__ float tile_amax[16][33];
    const int64_t KB = K >> 4;
    const uint32_t kb_tiles = (uint32_t)((KB + 31) >> 5);
    const uint32_t tiles = (uint32_t)(M >> 4) * kb_tiles;
    const bool pack4 = (KB & 3) == 0;
    const float s_g = global_scale_of(*amax_ptr);
    if (write_gs && blockIdx.x == 0 && threadIdx.x == 0) *gs_out = s_g;
    uint32_t sw[8];
    rht_sign_words(mask, sw);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (uint32_t t = blockIdx.x; t < tiles; t += gridDim.x) {
        const uint32_t rt = t / kb_tiles, kt = t - rt * kb_tiles;
        const int64_t row = (int64_t)rt * 16 + w;
        const int64_t kb = (int64_t)kt * 32 + lane;
        const bool valid = kb < KB;
        f32x2 P[8];
        if (valid) {
            const uint16_t *p = x + row * ldx + kb * 16;
            if (RHT) load_rht16(p, sw, P);
            else load16_pairs(p, P);
        } else {
#pragma unroll
            for (int k = 0; k < 8; k++) P[k] = 0ull;
        }
        const float bamax = pairs_absmax(P);
        tile_amax[w][lane] = bamax;
        __syncthreads();
        float tmax = 0.0f;
#pragma unroll
        for (int r = 0; r < 16; r++) tmax = fmaxf(tmax, tile_amax[r][lane]);
        __syncthreads();
        NvCand c = nv_candidate(P, tmax, 6.0f, s_g);
        if (valid) *reinterpret_cast<uint2 *>(codes + row * (K >> 1) + kb * 8) = c.codes;
        store_sf(sf, valid, c.sb, row, kb, KB, pack4);
    }
}

// ===================================================================== MXFP8
// E8M0 exponent of a block: clamp(floor(log2 amax) - 8, -127, 127).
BSQ_DEV int mx_exponent(float bamax) {
    int E = floor_log2(bamax) - 8;
    return E < -127 ? -127 : (E > 127 ? 127 : E);
}

// Quantize 8 consecutive outputs of one block (E known); idx0 is the output
// linear index of v[0] (a multiple of 8).  Returns 8 codes packed in uint2.
template <bool SR>
BSQ_DEV uint2 mx_encode8(const float v[8], bool zero_block, int E, uint64_t idx0, uint32_t seed_lo,
                         uint32_t seed_hi, uint32_t stream_id) {
    if (zero_block) return make_uint2(0u, 0u);
    const float inv = exp2i(-E);
    float s[8];
#pragma unroll
    for (int i = 0; i < 8; i++) s[i] = fminf(fmaxf(__fmul_rn(v[i], inv), -448.0f), 448.0f);
    uint32_t c[8];
    if (SR) {
        const uint64_t g = idx0 >> 3;
        uint4 r = philox4x32_10(make_uint4((uint32_t)g, (uint32_t)(g >> 32), stream_id, 0u), seed_lo, seed_hi);
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 8; i++) c[i] = e4m3_sr(s[i], (i & 1) ? (w[i >> 1] >> 16) : (w[i >> 1] & 0xFFFFu));
    } else {
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            uint32_t p = cvt_e4m3x2(s[i], s[i + 1]);
            c[i] = p & 0xFFu;
            c[i + 1] = p >> 8;
        }
    }
    return make_uint2(c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24),
                      c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24));
}

// Row-wise: one thread per 8 elements, 4 lanes per block of 32.
template <bool SR>
__global__ void __launch_bounds__(256) quant_mxfp8_row_kernel(
    const uint16_t *__restrict__ x, int64_t M, int64_t K, int64_t ldx, uint32_t seed_lo, uint32_t seed_hi,
    uint32_t stream_id, uint8_t *__restrict__ codes, uint8_t *__restrict__ sf, RowMap map) {
    const int64_t K8 = K >> 3, KB = K >> 5;
    const bool pack4 = (KB & 3) == 0;
    const int lane = threadIdx.x & 31;
    const int lpr = 1 << map.lpr_shift;
    const int rpi = 256 >> map.lpr_shift;
    const int sub = threadIdx.x >> map.lpr_shift, lk = threadIdx.x & (lpr - 1);
    for (int64_t r0 = (int64_t)blockIdx.x * rpi; r0 < M; r0 += (int64_t)gridDim.x * rpi) {
        const int64_t row = r0 + sub;
        const bool row_ok = row < M;
        const int64_t rr = row_ok ? row : M - 1;
        for (int64_t c0 = 0; c0 < K8; c0 += lpr) {
            const int64_t c8 = c0 + lk;
            const bool valid = row_ok && c8 < K8;
            const int64_t cc = c8 < K8 ? c8 : K8 - 1;
            float v[8];
            load8_bf16(x + rr * ldx + cc * 8, v);
            float m = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; i++) m = fmaxf(m, fabsf(v[i]));
            m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
            m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
            const bool zero = (m == 0.0f);
            const int E = zero ? 0 : mx_exponent(m);
            const uint64_t idx0 = (uint64_t)(rr * K + cc * 8);
            uint2 q = mx_encode8<SR>(v, zero, E, idx0, seed_lo, seed_hi, stream_id);
            if (valid) *reinterpret_cast<uint2 *>(codes + rr * K + cc * 8) = q;
            // scale byte: lanes 4j hold block j; 4 blocks (16 lanes) per word
            const uint32_t sb = zero ? 0u : (uint32_t)(E + 127);
            const int64_t kb = cc >> 2;
            if (pack4) {
                uint32_t b1 = __shfl_down_sync(0xFFFFFFFFu, sb, 4);
                uint32_t b2 = __shfl_down_sync(0xFFFFFFFFu, sb, 8);
                uint32_t b3 = __shfl_down_sync(0xFFFFFFFFu, sb, 12);
                if (valid && (lane & 15) == 0)
                    *reinterpret_cast<uint32_t *>(sf + sf_word_offset(rr, kb >> 2, KB)) =
                        sb | (b1 << 8) | (b2 << 16) | (b3 << 24);
            } else if (valid && (lane & 3) == 0) {
                sf[sf_offset(rr, kb, KB)] = (uint8_t)sb;
            }
        }
    }
}

// Column-wise (output = quantization of the transpose), from bf16 or from
// row-wise MXFP8 (dequantized exactly).  A CTA tile covers 128 input rows
// (output columns) x 64 input columns (output rows); shared memory holds the
// tile as fp32 [64][128], written with lanes along m (conflict-free) and read
// as 8 consecutive m per thread.
constexpr int CT_M = 128, CT_K = 64;

template <bool FROM_MX, bool SR>
__global__ void __launch_bounds__(256) quant_mxfp8_col_kernel(
    const void *__restrict__ xin, const uint8_t *__restrict__ sf_in, int64_t M, int64_t K, int64_t ldx,
    uint32_t seed_lo, uint32_t seed_hi, uint32_t stream_id, uint8_t *__restrict__ codes,
    uint8_t *__restrict__ sf) {
    __shared__ __align__(16) float tile[CT_K][CT_M];
    const uint32_t m_tiles = (uint32_t)((M + CT_M - 1) / CT_M), k_tiles = (uint32_t)((K + CT_K - 1) / CT_K);
    const int64_t MB = M >> 5;  // output blocks per output row
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (uint32_t t = blockIdx.x; t < m_tiles * k_tiles; t += gridDim.x) {
        const uint32_t kt = t / m_tiles, mt = t - kt * m_tiles;
        const int64_t m0 = (int64_t)mt * CT_M, k0 = (int64_t)kt * CT_K;
        // ---- load: each thread reads 32 contiguous bytes of one input row
        if (!FROM_MX) {
            const uint16_t *x = static_cast<const uint16_t *>(xin);
#pragma unroll
            for (int it = 0; it < 2; it++) {
                const int task = warp + 8 * it;  // 16 tasks of (row block of 32, chunk of 16 k)
                const int ml = (task & 3) * 32 + lane;
                const int kc = task >> 2;         // 0..3, 16 k each
                const int64_t m = m0 + ml, k = k0 + kc * 16;
                float v[16];
                if (m < M && k < K) {  // K % 8 == 0; a chunk may be half valid
                    load8_bf16(x + m * ldx + k, v);
                    if (k + 8 < K) load8_bf16(x + m * ldx + k + 8, v + 8);
                    else
#pragma unroll
                        for (int i = 8; i < 16; i++) v[i] = 0.0f;
                } else {
#pragma unroll
                    for (int i = 0; i < 16; i++) v[i] = 0.0f;
                }
#pragma unroll
                for (int i = 0; i < 16; i++) tile[kc * 16 + i][ml] = v[i];
            }
        } else {
            const uint8_t *x = static_cast<const uint8_t *>(xin);
            const int64_t KBin = K >> 5;
            const int ml = (warp & 3) * 32 + lane;
            const int kc = warp >> 2;  // 0..1, 32 k each
            const int64_t m = m0 + ml, k = k0 + kc * 32;
            float v[32];
            if (m < M && k < K) {
                const float sc = exp2i((int)__ldg(sf_in + sf_offset(m, k >> 5, KBin)) - 127);
                const uint4 *p = reinterpret_cast<const uint4 *>(x + m * ldx + k);
                uint4 a = __ldg(p), b = __ldg(p + 1);
                const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
                for (int i = 0; i < 8; i++) {
                    float f0, f1, f2, f3;
                    e4m3x2_to_f32(w[i] & 0xFFFFu, f0, f1);
                    e4m3x2_to_f32(w[i] >> 16, f2, f3);
                    v[4 * i] = __fmul_rn(f0, sc);
                    v[4 * i + 1] = __fmul_rn(f1, sc);
                    v[4 * i + 2] = __fmul_rn(f2, sc);
                    v[4 * i + 3] = __fmul_rn(f3, sc);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; i++) v[i] = 0.0f;
            }
#pragma unroll
            for (int i = 0; i < 32; i++) tile[kc * 32 + i][ml] = v[i];
        }
        __syncthreads();
        // ---- quantize: 64 output rows x 16 chunks of 8; 4 lanes per block
#pragma unroll
        for (int it = 0; it < 4; it++) {
            const int task = threadIdx.x + 256 * it;
            const int mc = task & 15, kl = task >> 4;
            const int64_t k = k0 + kl, m = m0 + mc * 8;
            const float4 *src = reinterpret_cast<const float4 *>(&tile[kl][mc * 8]);
            float4 a = src[0], b = src[1];
            float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            float am = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; i++) am = fmaxf(am, fabsf(v[i]));
            am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
            am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 2));
            const bool zero = (am == 0.0f);
            const int E = zero ? 0 : mx_exponent(am);
            const bool valid = (k < K) && (m < M);
            const uint64_t idx0 = (uint64_t)(k * M + m);
            uint2 q = mx_encode8<SR>(v, zero, E, idx0, seed_lo, seed_hi, stream_id);
            if (valid) *reinterpret_cast<uint2 *>(codes + k * M + m) = q;
            const uint32_t sb = zero ? 0u : (uint32_t)(E + 127);
            // lanes with mc = 0, 4, 8, 12 hold blocks 0..3 of this tile row
            uint32_t b1 = __shfl_down_sync(0xFFFFFFFFu, sb, 4);
            uint32_t b2 = __shfl_down_sync(0xFFFFFFFFu, sb, 8);
            uint32_t b3 = __shfl_down_sync(0xFFFFFFFFu, sb, 12);
            const int64_t blk = m >> 5;
            if (k < K && (mc & 3) == 0 && m < M) {
                if (m0 + CT_M <= M && (MB & 3) == 0) {
                    if (mc == 0)
                        *reinterpret_cast<uint32_t *>(sf + sf_word_offset(k, blk >> 2, MB)) =
                            sb | (b1 << 8) | (b2 << 16) | (b3 << 24);
                } else {
                    sf[sf_offset(k, blk, MB)] = (uint8_t)sb;
                }
            }
        }
        __syncthreads();
    }
}

// ===================================================================== RHT
__global__ void __launch_bounds__(256) rht_kernel(const uint16_t *__restrict__ x, uint16_t *y, int64_t M,
                                                  int64_t K, int64_t ldx, int64_t ldy, uint32_t mask, RowMap map) {
    const int64_t KB = K >> 4;
    uint32_t sw[8];
    rht_sign_words(mask, sw);
    const int lpr = 1 << map.lpr_shift;
    const int rpi = 256 >> map.lpr_shift;
    const int sub = threadIdx.x >> map.lpr_shift, lk = threadIdx.x & (lpr - 1);
    for (int64_t r0 = (int64_t)blockIdx.x * rpi; r0 < M; r0 += (int64_t)gridDim.x * rpi) {
        const int64_t row = r0 + sub;
        if (row >= M) continue;
        for (int64_t kb = lk; kb < KB; kb += lpr) {
            f32x2 P[8];
            load_rht16(x + row * ldx + kb * 16, sw, P);
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 8; i++) {
                float a, b;
                f2_unpack(P[i], a, b);
                __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
                w[i] = *reinterpret_cast<uint32_t *>(&h);
            }
            uint4 *q = reinterpret_cast<uint4 *>(y + row * ldy + kb * 16);
            q[0] = make_uint4(w[0], w[1], w[2], w[3]);
            q[1] = make_uint4(w[4], w[5], w[6], w[7]);
        }
    }
}

// ===================================================================== launchers
static int grid_for(int64_t work_items, int per_block, int max_ctas) {
    int64_t g = (work_items + per_block - 1) / per_block;
    if (g > max_ctas) g = max_ctas;
    return (int)(g < 1 ? 1 : g);
}

void launch_amax(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, bool rht, uint32_t mask,
                 const int32_t *row_index, unsigned int *amax_bits, int num_sms, cudaStream_t s) {
    RowMap map{lpr_shift_for(K >> 4)};
    const int grid = grid_for(M, 256 >> map.lpr_shift, num_sms * 8);
#define BSQ_AMAX(R, G) amax_kernel<R, G><<<grid, 256, 0, s>>>(x, M, K, ldx, mask, row_index, amax_bits, map)
    if (rht) { if (row_index) BSQ_AMAX(true, true); else BSQ_AMAX(true, false); }
    else { if (row_index) BSQ_AMAX(false, true); else BSQ_AMAX(false, false); }
#undef BSQ_AMAX
}

void launch_finalize_global_scale(float *gs, cudaStream_t s) { finalize_global_scale_kernel<<<1, 1, 0, s>>>(gs); }

void launch_quant_nvfp4(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, bool block_2d, bool fos,
                        bool rht, uint32_t mask, const int32_t *row_index, int G, const int32_t *row_off,
                        const int32_t *sf_off, const float *amax_ptr, float *gs_out, bool write_gs,
                        uint8_t *codes, uint8_t *sf, int num_sms, cudaStream_t s) {
    if (block_2d) {
        const int64_t tiles = (M >> 4) * (((K >> 4) + 31) >> 5);
        const int grid = grid_for(tiles, 1, num_sms * 4);
        if (rht)
            quant_nvfp4_2d_kernel<true><<<grid, 512, 0, s>>>(x, M, K, ldx, mask, amax_ptr, gs_out, write_gs, codes, sf);
        else
            quant_nvfp4_2d_kernel<false><<<grid, 512, 0, s>>>(x, M, K, ldx, mask, amax_ptr, gs_out, write_gs, codes, sf);
        return;
    }
    RowMap map{lpr_shift_for(K >> 4)};
    const int grid = grid_for(M, 256 >> map.lpr_shift, num_sms * 8);
    const bool gather = row_index != nullptr, grouped = G > 0;
#define BSQ_NV1(R, F, GA, GR)                                                                            \
    quant_nvfp4_1d_kernel<R, F, GA, GR><<<grid, 256, 0, s>>>(x, M, K, ldx, mask, row_index, G, row_off, \
                                                            sf_off, amax_ptr, gs_out, write_gs, codes, sf, map)
#define BSQ_NV1_G(R, F)                                 \
    do {                                                \
        if (gather) {                                   \
            if (grouped) BSQ_NV1(R, F, true, true);     \
            else BSQ_NV1(R, F, true, false);            \
        } else {                                        \
            if (grouped) BSQ_NV1(R, F, false, true);    \
            else BSQ_NV1(R, F, false, false);           \
        }                                               \
    } while (0)
    if (rht) { if (fos) BSQ_NV1_G(true, true); else BSQ_NV1_G(true, false); }
    else { if (fos) BSQ_NV1_G(false, true); else BSQ_NV1_G(false, false); }
#undef BSQ_NV1_G
#undef BSQ_NV1
}

void launch_quant_mxfp8(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, bool colwise, bool sr,
                        uint64_t seed, uint32_t stream_id, uint8_t *codes, uint8_t *sf, int num_sms,
                        cudaStream_t s) {
    const uint32_t lo = (uint32_t)seed, hi = (uint32_t)(seed >> 32);
    if (!colwise) {
        RowMap map{lpr_shift_for(K >> 3)};
        if (map.lpr_shift < 2) map.lpr_shift = 2;  // 4 lanes per block of 32
        const int grid = grid_for(M, 256 >> map.lpr_shift, num_sms * 8);
        if (sr) quant_mxfp8_row_kernel<true><<<grid, 256, 0, s>>>(x, M, K, ldx, lo, hi, stream_id, codes, sf, map);
        else quant_mxfp8_row_kernel<false><<<grid, 256, 0, s>>>(x, M, K, ldx, lo, hi, stream_id, codes, sf, map);
        return;
    }
    const int64_t tiles = ((M + CT_M - 1) / CT_M) * ((K + CT_K - 1) / CT_K);
    const int grid = grid_for(tiles, 1, num_sms * 6);
    if (sr)
        quant_mxfp8_col_kernel<false, true><<<grid, 256, 0, s>>>(x, nullptr, M, K, ldx, lo, hi, stream_id, codes, sf);
    else
        quant_mxfp8_col_kernel<false, false><<<grid, 256, 0, s>>>(x, nullptr, M, K, ldx, lo, hi, stream_id, codes, sf);
}

void launch_requant_transpose(const uint8_t *codes_row, const uint8_t *sf_row, int64_t M, int64_t K, bool sr,
                              uint64_t seed, uint32_t stream_id, uint8_t *codes_col, uint8_t *sf_col,
                              int num_sms, cudaStream_t s) {
    const uint32_t lo = (uint32_t)seed, hi = (uint32_t)(seed >> 32);
    const int64_t tiles = ((M + CT_M - 1) / CT_M) * ((K + CT_K - 1) / CT_K);
    const int grid = grid_for(tiles, 1, num_sms * 6);
    if (sr)
        quant_mxfp8_col_kernel<true, true><<<grid, 256, 0, s>>>(codes_row, sf_row, M, K, K, lo, hi, stream_id,
                                                                codes_col, sf_col);
    else
        quant_mxfp8_col_kernel<true, false><<<grid, 256, 0, s>>>(codes_row, sf_row, M, K, K, lo, hi, stream_id,
                                                                 codes_col, sf_col);
}

void launch_rht(const uint16_t *x, uint16_t *y, int64_t M, int64_t K, int64_t ldx, int64_t ldy, uint32_t mask,
                int num_sms, cudaStream_t s) {
    RowMap map{lpr_shift_for(K >> 4)};
    const int grid = grid_for(M, 256 >> map.lpr_shift, num_sms * 8);
    rht_kernel<<<grid, 256, 0, s>>>(x, y, M, K, ldx, ldy, mask, map);
}

}  // namespace bsq
