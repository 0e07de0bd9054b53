// nvfp4.cuh -- the NVFP4 block arithmetic shared by the quantize kernels and
// the GEMM's quantizing epilogue: the global scale, block maxima (optionally
// of the RHT output), the E4M3 block-scale code, E2M1 codes, the Four Over
// Six choice, and the swizzled scale-factor store.  Every step that decides a
// code is an explicit round-to-nearest intrinsic or PTX instruction, so the
// results do not depend on the file's contraction settings.
#pragma once
#include <cstdint>

#include "common.cuh"

namespace bsq {

// s_g = amax / (6 * 448); amax == 0 gives 1.
BSQ_DEV float global_scale_of(float amax) { return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 2688.0f); }

// max |y| of one 16-element block: with the RHT, y = u / 4 exactly and
// RN(u/4) is monotone in u, so max|y| = RN(max|u| / 4): the quarter is
// applied once, to the maximum.
template <bool RHT>
BSQ_DEV float block_absmax(const uint32_t w[8], const uint32_t sw[8]) {
    if (RHT) return __fmul_rn(rht16_u_absmax(w, sw), 0.25f);
    f32x2 P[8];
    words_to_pairs(w, P);
    return pairs_absmax3(P);
}

// Per-CTA tables and constants of one tensor's global scale s_g.  For every
// E4M3 scale code sb: den[sb] = RN(e4m3(sb) * s_g) and rcp[sb] = RN(1/den)
// -- the same two operations each block would do, done once.  The block
// scale t = RN(RN(bamax / 6) / s_g) is first estimated as RN(bamax * c6),
// c6 = RN(1 / RN(6 s_g)); the estimate is within 5 ulps of t, so wherever
// it lies more than 16 ulps from every E4M3 rounding boundary it rounds to
// the same code, and everywhere else (or outside the ranges where the bound
// holds) the exact two divisions are done.
struct NvScale {
    float s_g, c6, c4;
    bool fast;  // s_g in [2^-90, 2^100]: the estimate bound and the exact 1/4 fold hold
};

BSQ_DEV NvScale nv_scale_setup(float s_g, float *den_tab, float *rcp_tab) {
    if (threadIdx.x < 128) {
        const float den = __fmul_rn(e4m3_to_f32(threadIdx.x), s_g);
        den_tab[threadIdx.x] = den;
        rcp_tab[threadIdx.x] = (threadIdx.x == 0 || threadIdx.x == 127) ? 0.0f : __frcp_rn(den);
    }
    __syncthreads();
    NvScale c;
    c.s_g = s_g;
    c.c6 = __frcp_rn(__fmul_rn(6.0f, s_g));
    c.c4 = __frcp_rn(__fmul_rn(4.0f, s_g));
    c.fast = s_g >= 0x1p-90f && s_g <= 0x1p100f;
    return c;
}

// E4M3 code of RN(RN(bamax / divisor) / s_g) (satfinite, RNE).
BSQ_DEV uint32_t nv_scale_code(float bamax, float divisor, float c_div, const NvScale &c) {
    if (c.fast && bamax >= 0x1p-120f) {
        const float te = __fmul_rn(bamax, c_div);
        const int lowd = (int)(__float_as_uint(te) & 0xFFFFFu) - 0x80000;
        if (te >= 0x1p-6f && (lowd > 16 || lowd < -16)) return e4m3_rne(te);
    }
    return e4m3_rne(__fdiv_rn(__fdiv_rn(bamax, divisor), c.s_g));
}

// E2M1 codes of q = y * r for one block given as u (RHT: y = u / 4) or y.
// With the fold, q = RN(u * (r / 4)), equal to RN(RN(u / 4) * r) whenever
// u / 4 is not subnormal; when it is, |q| < 2^-27 (r <= 2^99 for s_g >=
// 2^-90) and both give the zero code.
template <bool RHT>
BSQ_DEV uint2 nv_codes(const f32x2 P[8], float r, bool fold) {
    float rr = r;
    f32x2 Q[8];
#pragma unroll
    for (int k = 0; k < 8; k++) Q[k] = P[k];
    if (RHT) {
        if (fold) rr = __fmul_rn(r, 0.25f);
        else pairs_scale(Q, 0.25f);
    }
    const f32x2 R = f2_pack(rr, rr);
    float q[16];
#pragma unroll
    for (int k = 0; k < 8; k++) f2_unpack(f2_mul(Q[k], R), q[2 * k], q[2 * k + 1]);
    return make_uint2(cvt_e2m1x8(q), cvt_e2m1x8(q + 8));
}

// Squared error of a candidate (scale den, codes), summed pairwise (0+1),
// (2+3), ... over four levels, on the block values y.  Scalar IEEE
// intrinsics throughout: the compiler may fuse a packed mul.rn.f32x2 with a
// following sub.rn.f32x2 into one rounding (seen on a block whose two
// candidates tie exactly), and __fmul_rn / __fsub_rn are never fused.
BSQ_DEV float nv_block_err(const f32x2 Y[8], uint2 codes, float den) {
    float v[16], dec[16];
#pragma unroll
    for (int k = 0; k < 8; k++) f2_unpack(Y[k], v[2 * k], v[2 * k + 1]);
    e2m1x8_to_f32(codes.x, dec);
    e2m1x8_to_f32(codes.y, dec + 8);
    float e[16];
#pragma unroll
    for (int i = 0; i < 16; i++) {
        const float d = __fsub_rn(v[i], __fmul_rn(dec[i], den));
        e[i] = __fmul_rn(d, d);
    }
#pragma unroll
    for (int w = 16; w > 1; w >>= 1)
#pragma unroll
        for (int i = 0; i < w / 2; i++) e[i] = __fadd_rn(e[2 * i], e[2 * i + 1]);
    return e[0];
}

// One 1x16 block: scale code and packed codes (Four Over Six optional).
template <bool RHT, bool FOS>
BSQ_DEV void nv_block_1d(const uint32_t w[8], const uint32_t sw[8], const NvScale &c, const float *den_tab,
                         const float *rcp_tab, uint32_t &sb, uint2 &codes) {
    f32x2 P[8];
    if (RHT) rht16_u_words(w, sw, P);
    else words_to_pairs(w, P);
    const float mu = pairs_absmax3(P);
    const float bamax = RHT ? __fmul_rn(mu, 0.25f) : mu;
    sb = nv_scale_code(bamax, 6.0f, c.c6, c);
    codes = sb ? nv_codes<RHT>(P, rcp_tab[sb], c.fast) : make_uint2(0u, 0u);
    if (FOS) {
        const uint32_t sb4 = nv_scale_code(bamax, 4.0f, c.c4, c);
        const uint2 codes4 = sb4 ? nv_codes<RHT>(P, rcp_tab[sb4], c.fast) : make_uint2(0u, 0u);
        if (RHT) pairs_scale(P, 0.25f);  // the block values y for the error
        if (nv_block_err(P, codes4, den_tab[sb4]) < nv_block_err(P, codes, den_tab[sb])) {
            sb = sb4;
            codes = codes4;
        }
    }
}

// Writes the scale byte of a unit: packs 4 consecutive blocks into one word
// when the row's block count is a multiple of 4 (lanes 4j..4j+3 hold blocks
// 4i..4i+3 of one row), else stores the byte.  The offset is computed in the
// index type I (uint32_t where the scale buffer holds fewer than 2^31 bytes);
// sf_row is read only when valid.
template <typename I>
BSQ_DEV void store_sf_t(uint8_t *sf, bool valid, uint32_t sb, I sf_row, I kb, I KB, bool pack4) {
    if (pack4) {
        uint32_t b1 = __shfl_down_sync(0xFFFFFFFFu, sb, 1);
        uint32_t b2 = __shfl_down_sync(0xFFFFFFFFu, sb, 2);
        uint32_t b3 = __shfl_down_sync(0xFFFFFFFFu, sb, 3);
        if (valid && (threadIdx.x & 3) == 0) {
            uint32_t w = (sb & 0xFFu) | ((b1 & 0xFFu) << 8) | ((b2 & 0xFFu) << 16) | ((b3 & 0xFFu) << 24);
            *reinterpret_cast<uint32_t *>(sf + (size_t)sf_word_offset_t<I>(sf_row, kb >> 2, KB)) = w;
        }
    } else if (valid) {
        sf[(size_t)sf_offset_t<I>(sf_row, kb, KB)] = (uint8_t)sb;
    }
}

}  // namespace bsq
