// common.cuh -- device helpers shared by the libbsq kernels: number-format
// conversions (hand-written PTX cvt), Philox4x32-10, the MMA scale-factor
// layout, the per-device error word.  Every floating-point step that decides
// a code uses an explicit round-to-nearest intrinsic so that the compiler
// cannot contract or reorder it.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/bsq.h"

#define BSQ_DEV __device__ __forceinline__

namespace bsq {

// ---------------------------------------------------------------- launch overlap
// Programmatic dependent launch.  A kernel launched by launch_dependent() may
// be scheduled while the kernel before it in the stream is still running.
// Every such kernel calls grid_dependency_wait() before its first access to
// global memory: the call returns once the previous kernel has completed and
// its writes are visible, so results are those of plain stream order and
// only the launch latency overlaps.  grid_dependents_launch() lets the next
// kernel be scheduled as soon as every CTA of this one has called it (or has
// exited).  Outside such launches both are no-ops.
BSQ_DEV void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
BSQ_DEV void grid_dependents_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Current value of a kernel-selection override (BSQ_KNOB_*; -1 = automatic).
int kernel_choice(int knob);

// kern<<<grid, block, smem, s>>>(args...), marked for programmatic dependent
// launch unless BSQ_KNOB_LAUNCH_OVERLAP is 0.  kern must call
// grid_dependency_wait() before it touches global memory.
template <class... P, class... A>
cudaError_t launch_dependent(void (*kern)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             A &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = kernel_choice(BSQ_KNOB_LAUNCH_OVERLAP) != 0 ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<A &&>(args)...);
}

// ---------------------------------------------------------------- error word
// One 32-bit word per device: bit 0 set by a bounded wait that ran out, bits
// 8..15 hold the site id of the first such wait.
struct ErrWord {
    unsigned int *ptr;
};

BSQ_DEV void report_timeout(unsigned int *err, unsigned int site) {
    if (err) atomicOr(err, 1u | ((site & 0xFFu) << 8));
}

BSQ_DEV uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Sets cudaFuncAttributeMaxDynamicSharedMemorySize of `kern` to `bytes` on
// the current device, once per (kernel, device); BSQ_OK or BSQ_ERR_CUDA.
int smem_attr_once(const void *kern, int bytes);

// ---------------------------------------------------------------- bf16
BSQ_DEV float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
BSQ_DEV float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// 16-byte streaming load of 8 bf16 -> 8 fp32
BSQ_DEV void load8_bf16(const uint16_t *p, float v[8]) {
    uint4 q = __ldg(reinterpret_cast<const uint4 *>(p));
    v[0] = bf16_lo(q.x); v[1] = bf16_hi(q.x);
    v[2] = bf16_lo(q.y); v[3] = bf16_hi(q.y);
    v[4] = bf16_lo(q.z); v[5] = bf16_hi(q.z);
    v[6] = bf16_lo(q.w); v[7] = bf16_hi(q.w);
}

// ---------------------------------------------------------------- E4M3 / E2M1
// cvt.rn.satfinite.e4m3x2.f32: the first source lands in the upper byte.
BSQ_DEV uint32_t cvt_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

BSQ_DEV uint32_t e4m3_rne(float v) { return cvt_e4m3x2(v, 0.0f) & 0xFFu; }

// E4M3 byte -> fp32 (exact), via cvt.rn.f16x2.e4m3x2 (low byte -> low half).
BSQ_DEV float e4m3_to_f32(uint32_t code) {
    uint32_t h2;
    uint16_t in = (uint16_t)(code & 0xFFu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    __half_raw hr;
    hr.x = (unsigned short)(h2 & 0xFFFFu);
    return __half2float(__half(hr));
}

// Two E4M3 bytes (low, high of a 16-bit word) -> two fp32.
BSQ_DEV void e4m3x2_to_f32(uint32_t two, float &lo, float &hi) {
    uint32_t h2;
    uint16_t in = (uint16_t)(two & 0xFFFFu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    __half_raw a, b;
    a.x = (unsigned short)(h2 & 0xFFFFu);
    b.x = (unsigned short)(h2 >> 16);
    lo = __half2float(__half(a));
    hi = __half2float(__half(b));
}

// 8 fp32 -> 8 E2M1 nibbles, element 2j in the low nibble of byte j.
// cvt.rn.satfinite.e2m1x2.f32 d, a, b puts a in the upper nibble.
BSQ_DEV uint32_t cvt_e2m1x8(const float q[8]) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(q[0]), "f"(q[1]), "f"(q[2]), "f"(q[3]), "f"(q[4]), "f"(q[5]), "f"(q[6]), "f"(q[7]));
    return out;
}

// Eight E2M1 codes (packed as by cvt_e2m1x8: element 2i in the low nibble of
// byte i) -> fp32, exactly, through cvt.rn.f16x2.e2m1x2 (every E2M1 value is
// an f16 and an fp32 value; -0 stays -0).
BSQ_DEV void e2m1x8_to_f32(uint32_t w, float v[8]) {
    uint32_t h[4];
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(w));
#pragma unroll
    for (int i = 0; i < 4; i++) {
        __half_raw lo, hi;
        lo.x = (unsigned short)(h[i] & 0xFFFFu);
        hi.x = (unsigned short)(h[i] >> 16);
        v[2 * i] = __half2float(__half(lo));
        v[2 * i + 1] = __half2float(__half(hi));
    }
}

// The two E2M1 codes in the low byte of w (element 0 in the low nibble) ->
// fp32, exactly, as e2m1x8_to_f32 does.
BSQ_DEV void e2m1x2_to_f32(uint32_t w, float &lo, float &hi) {
    uint32_t h;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t}"
        : "=r"(h)
        : "r"(w));
    __half_raw l, u;
    l.x = (unsigned short)(h & 0xFFFFu);
    u.x = (unsigned short)(h >> 16);
    lo = __half2float(__half(l));
    hi = __half2float(__half(u));
}

// floor(log2 a) for a finite a > 0 (normal or subnormal binary32).
BSQ_DEV int floor_log2(float a) {
    uint32_t b = __float_as_uint(a) & 0x7FFFFFFFu;
    int e = (int)(b >> 23);
    if (e) return e - 127;
    return (31 - __clz((int)b)) - 149;
}

// 2^k as a binary32 for k in [-149, 127].
BSQ_DEV float exp2i(int k) {
    if (k >= -126) return __uint_as_float((uint32_t)(k + 127) << 23);
    return __uint_as_float(1u << (k + 149));
}

// ---------------------------------------------------------------- Philox
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11): ten rounds of two
// 32x32->64 multiplies (0xD2511F53, 0xCD9E8D57) and xors with the round keys.
// The ten round keys for key (k0, k1): round r uses
// (k0 + r 0x9E3779B9, k1 + r 0xBB67AE85) mod 2^32.  Computed once on the host
// and passed as a kernel parameter, so the rounds read them from the
// constant bank instead of recomputing the schedule per call.
struct PhiloxKeys {
    uint32_t k0[10], k1[10];
};
static inline PhiloxKeys philox_keys(uint32_t k0, uint32_t k1) {
    PhiloxKeys K;
    for (int r = 0; r < 10; r++) {
        K.k0[r] = k0 + (uint32_t)r * 0x9E3779B9u;
        K.k1[r] = k1 + (uint32_t)r * 0xBB67AE85u;
    }
    return K;
}
BSQ_DEV uint4 philox4x32_10(uint4 c, const PhiloxKeys &K) {
#pragma unroll
    for (int r = 0; r < 10; r++) {
        const uint64_t p0 = (uint64_t)0xD2511F53u * c.x, p1 = (uint64_t)0xCD9E8D57u * c.z;
        c = make_uint4((uint32_t)(p1 >> 32) ^ c.y ^ K.k0[r], (uint32_t)p1, (uint32_t)(p0 >> 32) ^ c.w ^ K.k1[r],
                       (uint32_t)p0);
    }
    return c;
}

// Stochastic rounding of v (already clamped to +-448) to E4M3, with the
// 16-bit draw r16: round the magnitude up to the next E4M3 value iff
// r16 * 2^-16 < (|v| - lo) / ulp.
BSQ_DEV uint32_t e4m3_sr(float v, uint32_t r16) {
    uint32_t sgn = (__float_as_uint(v) >> 24) & 0x80u;
    float a = fabsf(v);
    if (a == 0.0f) return sgn;
    int fl = floor_log2(a);
    int ue = (fl > -6 ? fl : -6) - 3;
    float inv = exp2i(-ue), ulp = exp2i(ue);
    float lo = __fmul_rn(floorf(__fmul_rn(a, inv)), ulp);
    float frac = __fmul_rn(__fsub_rn(a, lo), inv);
    float u = __fmul_rn((float)r16, 1.0f / 65536.0f);
    float mag = (u < frac) ? __fadd_rn(lo, ulp) : lo;
    return sgn | e4m3_rne(mag);
}



// ---------------------------------------------------------------- fp32 pairs
// sm_100 executes two fp32 operations per instruction on a 64-bit register
// pair (add/sub/mul.rn.f32x2); each lane is an ordinary IEEE RN operation.
typedef unsigned long long f32x2;
BSQ_DEV f32x2 f2_pack(float lo, float hi) {
    f32x2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
BSQ_DEV void f2_unpack(f32x2 r, float &lo, float &hi) { asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r)); }
BSQ_DEV f32x2 f2_add(f32x2 a, f32x2 b) {
    f32x2 r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
BSQ_DEV f32x2 f2_sub(f32x2 a, f32x2 b) {
    f32x2 r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
BSQ_DEV f32x2 f2_mul(f32x2 a, f32x2 b) {
    f32x2 r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// ---------------------------------------------------------------- RHT
// Sign words for the 16-point RHT applied to packed bf16 pairs: word k flips
// element 2k (bit 15) and 2k+1 (bit 31) where the sign vector says s = -1.
BSQ_DEV void rht_sign_words(uint32_t mask, uint32_t sw[8]) {
#pragma unroll
    for (int k = 0; k < 8; k++) sw[k] = (((mask >> (2 * k)) & 1u) << 15) | (((mask >> (2 * k + 1)) & 1u) << 31);
}

// Loads 16 bf16 (two 16-byte loads), applies the signs and the Sylvester
// butterflies of stride 1, 2, 4, 8 (in that order, each an RN add or
// subtract) and the exact 1/4 scaling: y = 1/4 * H16 * diag(s) * x as 8 fp32
// pairs (element 2k in the low lane of pair k).
BSQ_DEV void load_rht16(const uint16_t *p, const uint32_t sw[8], f32x2 P[8]) {
    const uint4 q0 = __ldg(reinterpret_cast<const uint4 *>(p));
    const uint4 q1 = __ldg(reinterpret_cast<const uint4 *>(p + 8));
    const uint32_t w[8] = {q0.x ^ sw[0], q0.y ^ sw[1], q0.z ^ sw[2], q0.w ^ sw[3],
                           q1.x ^ sw[4], q1.y ^ sw[5], q1.z ^ sw[6], q1.w ^ sw[7]};
#pragma unroll
    for (int k = 0; k < 8; k++) {
        const float a = bf16_lo(w[k]), b = bf16_hi(w[k]);
        P[k] = f2_pack(__fadd_rn(a, b), __fsub_rn(a, b));  // stride 1
    }
#pragma unroll
    for (int h = 1; h < 8; h <<= 1) {  // strides 2, 4, 8 as pair strides 1, 2, 4
#pragma unroll
        for (int base = 0; base < 8; base += 2 * h) {
#pragma unroll
            for (int k = base; k < base + h; k++) {
                const f32x2 a = P[k], b = P[k + h];
                P[k] = f2_add(a, b);
                P[k + h] = f2_sub(a, b);
            }
        }
    }
    const f32x2 quarter = f2_pack(0.25f, 0.25f);
#pragma unroll
    for (int k = 0; k < 8; k++) P[k] = f2_mul(P[k], quarter);
}

// 16 bf16 as 8 32-bit words (element 2k in the low half of word k), two
// 16-byte loads.
BSQ_DEV void load_words16(const uint16_t *p, uint32_t w[8]) {
    const uint4 q0 = __ldg(reinterpret_cast<const uint4 *>(p));
    const uint4 q1 = __ldg(reinterpret_cast<const uint4 *>(p + 8));
    w[0] = q0.x; w[1] = q0.y; w[2] = q0.z; w[3] = q0.w;
    w[4] = q1.x; w[5] = q1.y; w[6] = q1.z; w[7] = q1.w;
}
BSQ_DEV void words_to_pairs(const uint32_t w[8], f32x2 P[8]) {
#pragma unroll
    for (int k = 0; k < 8; k++) P[k] = f2_pack(bf16_lo(w[k]), bf16_hi(w[k]));
}
// u = H16 * diag(s) * x from 8 words, without the final 1/4: the same sign
// flips and butterflies (strides 1, 2, 4, 8, RN) as load_rht16; y = u / 4.
BSQ_DEV void rht16_u_words(const uint32_t w_in[8], const uint32_t sw[8], f32x2 P[8]) {
#pragma unroll
    for (int k = 0; k < 8; k++) {
        const uint32_t w = w_in[k] ^ sw[k];
        const float a = bf16_lo(w), b = bf16_hi(w);
        P[k] = f2_pack(__fadd_rn(a, b), __fsub_rn(a, b));
    }
#pragma unroll
    for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
        for (int base = 0; base < 8; base += 2 * h) {
#pragma unroll
            for (int k = base; k < base + h; k++) {
                const f32x2 a = P[k], b = P[k + h];
                P[k] = f2_add(a, b);
                P[k + h] = f2_sub(a, b);
            }
        }
    }
}
// three-input max (sm_100)
BSQ_DEV float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
// max |u| over the 16 outputs of rht16_u_words, without forming them: the
// last butterfly (stride 8) maps each pair (a, b) to RN(a + b) and RN(a - b),
// and max(|RN(a + b)|, |RN(a - b)|) = RN(|a| + |b|) -- one of a + b, a - b
// has magnitude |a| + |b| exactly, the other no more, and RN is symmetric
// and monotone.  (A NaN pair contributes NaN either way, which the maxima
// below skip as the per-output maxima do.)
BSQ_DEV float rht16_u_absmax(const uint32_t w_in[8], const uint32_t sw[8]) {
    f32x2 P[8];
#pragma unroll
    for (int k = 0; k < 8; k++) {
        const uint32_t w = w_in[k] ^ sw[k];
        const float a = bf16_lo(w), b = bf16_hi(w);
        P[k] = f2_pack(__fadd_rn(a, b), __fsub_rn(a, b));
    }
#pragma unroll
    for (int h = 1; h < 4; h <<= 1) {  // strides 2 and 4 as pair strides 1 and 2
#pragma unroll
        for (int base = 0; base < 8; base += 2 * h) {
#pragma unroll
            for (int k = base; k < base + h; k++) {
                const f32x2 a = P[k], b = P[k + h];
                P[k] = f2_add(a, b);
                P[k + h] = f2_sub(a, b);
            }
        }
    }
    float s[8];
#pragma unroll
    for (int k = 0; k < 4; k++) {
        float a0, a1, b0, b1;
        f2_unpack(P[k], a0, a1);
        f2_unpack(P[k + 4], b0, b1);
        s[2 * k] = __fadd_rn(fabsf(a0), fabsf(b0));
        s[2 * k + 1] = __fadd_rn(fabsf(a1), fabsf(b1));
    }
    return fmax3(fmax3(s[0], s[1], s[2]), fmax3(s[3], s[4], s[5]), fmax3(s[6], s[7], 0.0f));
}
BSQ_DEV void pairs_scale(f32x2 P[8], float c) {
    const f32x2 C = f2_pack(c, c);
#pragma unroll
    for (int k = 0; k < 8; k++) P[k] = f2_mul(P[k], C);
}
// max |v| over 8 pairs, as a tree of three-input maxima
BSQ_DEV float pairs_absmax3(const f32x2 P[8]) {
    float v[16];
#pragma unroll
    for (int k = 0; k < 8; k++) f2_unpack(P[k], v[2 * k], v[2 * k + 1]);
    float m0 = fmax3(fabsf(v[0]), fabsf(v[1]), fabsf(v[2]));
    float m1 = fmax3(fabsf(v[3]), fabsf(v[4]), fabsf(v[5]));
    float m2 = fmax3(fabsf(v[6]), fabsf(v[7]), fabsf(v[8]));
    float m3 = fmax3(fabsf(v[9]), fabsf(v[10]), fabsf(v[11]));
    float m4 = fmax3(fabsf(v[12]), fabsf(v[13]), fabsf(v[14]));
    return fmax3(fmax3(m0, m1, m2), fmax3(m3, m4, fabsf(v[15])), 0.0f);
}




// ---------------------------------------------------------------- SF layout
// Byte offset of (row r, block b) in a swizzled SF buffer whose rows hold
// nblk blocks: 512-byte atoms of 128 rows x 4 blocks, row-tile major.
BSQ_DEV int64_t sf_offset(int64_t r, int64_t b, int64_t nblk) {
    int64_t bt = (nblk + 3) >> 2;
    return (((r >> 7) * bt + (b >> 2)) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2) + (b & 3);
}
// sf_offset in the index type I: uint32_t where the scale buffer holds fewer
// than 2^31 bytes, so that the offset takes single 32-bit instructions.
template <typename I>
BSQ_DEV I sf_offset_t(I r, I b, I nblk) {
    const I bt = (nblk + 3) >> 2;
    return (((r >> 7) * bt + (b >> 2)) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2) + (b & 3);
}
template <typename I>
BSQ_DEV I sf_word_offset_t(I r, I b4, I nblk) {
    const I bt = (nblk + 3) >> 2;
    return (((r >> 7) * bt + b4) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2);
}
// Offset of the 4-byte word holding blocks 4j..4j+3 of row r.
BSQ_DEV int64_t sf_word_offset(int64_t r, int64_t b4, int64_t nblk) {
    int64_t bt = (nblk + 3) >> 2;
    return (((r >> 7) * bt + b4) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2);
}

}  // namespace bsq
