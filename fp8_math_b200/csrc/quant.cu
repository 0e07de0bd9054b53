// quant.cu -- the codec kernels of libbsq (sm_100a):
//   tensor amax (optionally of the RHT output), NVFP4 quantize (1x16 with
//   optional Four Over Six, row gather and expert groups; 16x16 tiles; a
//   one-launch amax + quantize form; stochastic rounding of the elements),
//   MXFP8 quantize (row-wise, column-wise; RNE or Philox SR), dequantize ->
//   transpose -> requantize, MXFP4 quantize, and the standalone 16-point RHT.
// All of them stream bf16/fp8 from HBM with 16-byte vector loads, reduce the
// block amax with warp shuffles, and write packed codes plus scale factors
// directly in the swizzled layout the block-scaled MMA reads.

#include "common.cuh"
#include "devcache.h"
#include "nvfp4.cuh"
#include "quant.cuh"
#include "sm100.cuh"

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


// CTA max -> atomicMax on the float bits (non-negative floats order like
// their bit patterns).  With a counter, the last CTA to finish also turns
// the tensor amax into s_g and writes it to *gs_out (fence, count, fence:
// every other CTA's maximum is visible to the last one).
BSQ_DEV void block_reduce_atomic_max(float m, unsigned int *amax_bits, unsigned int *counter, float *gs_out) {
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    __shared__ float red[32];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float b = red[0];
        for (int i = 1; i < (int)(blockDim.x >> 5); i++) b = fmaxf(b, red[i]);
        atomicMax(amax_bits, __float_as_uint(b));
        if (counter) {
            __threadfence();
            if (atomicAdd(counter, 1u) == gridDim.x - 1) {
                __threadfence();
                const float amax = __uint_as_float(atomicOr(amax_bits, 0u));
                *gs_out = global_scale_of(amax);
            }
        }
    }
}

// Rows (optionally gathered through row_index) of a strided tensor.
template <bool RHT, bool GATHER>
__global__ void __launch_bounds__(256) amax_kernel(const uint16_t *__restrict__ x, int64_t M, int64_t K,
                                                   int64_t ldx, uint32_t mask,
                                                   const int32_t *__restrict__ row_index,
                                                   unsigned int *amax_bits, unsigned int *counter, float *gs_out,
                                                   RowMap map) {
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
            uint32_t w[8];
            load_words16(rp + kb * 16, w);
            m = fmaxf(m, block_absmax<RHT>(w, sw));
        }
    }
    block_reduce_atomic_max(m, amax_bits, counter, gs_out);
}

// Contiguous tensor as a flat sequence of 16-element blocks; four blocks per
// thread in flight (all loads issued before any is reduced).  I is the block
// index type: uint32_t when the block count and the loop's overshoot fit
// (below 2^31 blocks), which keeps the index arithmetic to single 32-bit
// instructions; int64_t otherwise.
template <bool RHT, typename I>
__global__ void __launch_bounds__(256) amax_flat_kernel(const uint16_t *__restrict__ x, int64_t nblk64, uint32_t mask,
                                                        unsigned int *amax_bits, unsigned int *counter,
                                                        float *gs_out) {
    grid_dependency_wait();
    grid_dependents_launch();
    uint32_t sw[8];
    rht_sign_words(mask, sw);
    const I nblk = (I)nblk64;
    const I stride = (I)gridDim.x * (I)blockDim.x;
    float m = 0.0f;
    for (I b = (I)blockIdx.x * (I)blockDim.x + (I)threadIdx.x; b < nblk; b += 4 * stride) {
        uint32_t w[4][8];
#pragma unroll
        for (int i = 0; i < 4; i++)
            if (b + i * stride < nblk) load_words16(x + (size_t)(b + i * stride) * 16, w[i]);
#pragma unroll
        for (int i = 0; i < 4; i++)
            if (b + i * stride < nblk) m = fmaxf(m, block_absmax<RHT>(w[i], sw));
    }
    block_reduce_atomic_max(m, amax_bits, counter, gs_out);
}


__global__ void finalize_global_scale_kernel(float *gs) { *gs = global_scale_of(*gs); }

// amax with one partial maximum per CTA in caller-given scratch (word 0: a
// CTA counter that must be zero on entry; word 1 + c: CTA c's maximum), for
// the no-allocation global-scale entry point.  CTA c covers the 16-element
// blocks [c * kPartialBlocks, (c + 1) * kPartialBlocks) of the row-major
// block sequence (row = b / (K / 16)); the last CTA to finish reduces the
// partials with all its threads and writes s_g.
template <bool RHT>
__global__ void __launch_bounds__(256) amax_partials_kernel(const uint16_t *__restrict__ x, int64_t M, int64_t K,
                                                            int64_t ldx, uint32_t mask, unsigned int *scratch,
                                                            float *gs_out) {
    uint32_t sw[8];
    rht_sign_words(mask, sw);
    const int64_t KB = K >> 4, nblk = M * KB;
    const int64_t b0 = (int64_t)blockIdx.x * kPartialBlocks;
    float m = 0.0f;
#pragma unroll 4
    for (int i = 0; i < kPartialBlocks / 256; i++) {
        const int64_t b = b0 + i * 256 + threadIdx.x;
        if (b < nblk) {
            const int64_t row = b / KB, kb = b - row * KB;
            uint32_t w[8];
            load_words16(x + row * ldx + kb * 16, w);
            m = fmaxf(m, block_absmax<RHT>(w, sw));
        }
    }
    __shared__ float red[8];
    __shared__ int last;
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float b = red[0];
        for (int i = 1; i < 8; i++) b = fmaxf(b, red[i]);
        scratch[1 + blockIdx.x] = __float_as_uint(b);
        __threadfence();
        last = atomicAdd(scratch, 1u) == gridDim.x - 1;
        if (last) __threadfence();
    }
    __syncthreads();
    if (!last) return;
    float a = 0.0f;
    for (unsigned int c = threadIdx.x; c < gridDim.x; c += 256) a = fmaxf(a, __uint_as_float(__ldcg(scratch + 1 + c)));
#pragma unroll
    for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, o));
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
    __syncthreads();
    if (threadIdx.x == 0) {
        float b = red[0];
        for (int i = 1; i < 8; i++) b = fmaxf(b, red[i]);
        *gs_out = global_scale_of(b);
    }
}

// ===================================================================== NVFP4
// Row -> scale-factor row under expert groups (binary search of offsets);
// -1 for a row outside [off[0], off[G]), which owns no scale-factor row.
BSQ_DEV int64_t grouped_sf_row(int64_t row, int G, const int32_t *__restrict__ off,
                               const int32_t *__restrict__ sfoff) {
    if (row < (int64_t)__ldg(off) || row >= (int64_t)__ldg(off + G)) return -1;
    int lo = 0, hi = G;  // off[lo] <= row < off[hi]
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if ((int64_t)__ldg(off + mid) <= row) lo = mid; else hi = mid;
    }
    return row - (int64_t)__ldg(off + lo) + (int64_t)__ldg(sfoff + lo);
}

// 1x16 blocks, rows (gathered, grouped): one thread per block of 16 (two
// 16-byte loads, one 8-byte code store).  Loops are warp-uniform so that
// shuffles see all lanes.
// I: the index type of the per-block offsets (uint32_t when the output holds
// fewer than 2^31 elements; a source row's start stays 64-bit).
template <bool RHT, bool FOS, bool GATHER, bool GROUPED, typename I>
__global__ void __launch_bounds__(256) quant_nvfp4_1d_kernel(
    const uint16_t *__restrict__ x, int64_t M, int64_t K, int64_t ldx, uint32_t mask,
    const int32_t *__restrict__ row_index, int G, const int32_t *__restrict__ row_off,
    const int32_t *__restrict__ sf_off, const float *scale_src, int src_is_amax, float *gs_out, int write_gs,
    uint8_t *__restrict__ codes, uint8_t *__restrict__ sf, RowMap map) {
    __shared__ float den_tab[128], rcp_tab[128];
    const int64_t KB = K >> 4;
    const bool pack4 = (KB & 3) == 0;
    const float s_g = src_is_amax ? global_scale_of(*scale_src) : *scale_src;
    if (write_gs && blockIdx.x == 0 && threadIdx.x == 0) *gs_out = s_g;
    const NvScale c = nv_scale_setup(s_g, den_tab, rcp_tab);
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
            uint32_t w[8];
            load_words16(rp + (size_t)((I)kk * 16), w);
            uint32_t sb;
            uint2 cd;
            nv_block_1d<RHT, FOS>(w, sw, c, den_tab, rcp_tab, sb, cd);
            if (valid) *reinterpret_cast<uint2 *>(codes + (size_t)((I)rr * (I)(K >> 1) + (I)kb * 8)) = cd;
            store_sf_t<I>(sf, valid && sf_row >= 0, sb, (I)(sf_row >= 0 ? sf_row : 0), (I)kb, (I)KB, pack4);
        }
    }
}

// 1x16 blocks of a contiguous tensor (ldx == K, no gather or groups) whose
// row holds a power-of-two number of blocks (>= 4): a flat sequence of
// blocks, two per thread in flight.  Lanes 4j..4j+3 hold four consecutive
// blocks of one row, so the scale bytes pack into one word.
template <bool RHT, bool FOS, typename I>
__global__ void __launch_bounds__(256) quant_nvfp4_1d_flat_kernel(
    const uint16_t *__restrict__ x, int64_t nblk64, int kb_shift, uint32_t mask, const float *scale_src,
    int src_is_amax, float *gs_out, int write_gs, uint8_t *__restrict__ codes, uint8_t *__restrict__ sf) {
    grid_dependency_wait();
    grid_dependents_launch();
    __shared__ float den_tab[128], rcp_tab[128];
    const float s_g = src_is_amax ? global_scale_of(*scale_src) : *scale_src;
    if (write_gs && blockIdx.x == 0 && threadIdx.x == 0) *gs_out = s_g;
    const NvScale c = nv_scale_setup(s_g, den_tab, rcp_tab);
    uint32_t sw[8];
    rht_sign_words(mask, sw);
    // I: the block index type (uint32_t below 2^31 blocks, as for amax_flat_kernel)
    const I nblk = (I)nblk64;
    const I KB = I(1) << kb_shift;
    const I bt = (KB + 3) >> 2;  // 4-block groups per row (the scale layout's atom columns)
    const I stride = (I)gridDim.x * (I)blockDim.x;
    // the loop bound is rounded to whole warps so that shuffles see all lanes
    const I nwarp_blk = (nblk + 31) & ~I(31);
    // scale bytes of lanes 4j..4j+3 (blocks 4i..4i+3 of one row) as one word
    // at the swizzled offset of (row, block group)
    auto store_sf4 = [&](bool valid, uint32_t sb, I b) {
        const uint32_t b1 = __shfl_down_sync(0xFFFFFFFFu, sb, 1);
        const uint32_t b2 = __shfl_down_sync(0xFFFFFFFFu, sb, 2);
        const uint32_t b3 = __shfl_down_sync(0xFFFFFFFFu, sb, 3);
        if (valid && (threadIdx.x & 3) == 0) {
            const I r = b >> kb_shift, b4 = (b & (KB - 1)) >> 2;
            const I off = (((r >> 7) * bt + b4) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2);
            *reinterpret_cast<uint32_t *>(sf + (size_t)off) =
                (sb & 0xFFu) | ((b1 & 0xFFu) << 8) | ((b2 & 0xFFu) << 16) | ((b3 & 0xFFu) << 24);
        }
    };
    for (I b = (I)blockIdx.x * (I)blockDim.x + (I)threadIdx.x; b - (I)(threadIdx.x & 31) < nwarp_blk;
         b += 2 * stride) {
        const I b1 = b + stride;
        const bool v0 = b < nblk, v1 = b1 < nblk;
        uint32_t w0[8], w1[8];
        load_words16(x + (size_t)(v0 ? b : 0) * 16, w0);
        load_words16(x + (size_t)(v1 ? b1 : 0) * 16, w1);
        uint32_t sb0, sb1;
        uint2 cd0, cd1;
        nv_block_1d<RHT, FOS>(w0, sw, c, den_tab, rcp_tab, sb0, cd0);
        if (v0) *reinterpret_cast<uint2 *>(codes + (size_t)b * 8) = cd0;
        store_sf4(v0, sb0, b);
        if (__any_sync(0xFFFFFFFFu, v1)) {
            nv_block_1d<RHT, FOS>(w1, sw, c, den_tab, rcp_tab, sb1, cd1);
            if (v1) *reinterpret_cast<uint2 *>(codes + (size_t)b1 * 8) = cd1;
            store_sf4(v1, sb1, b1);
        }
    }
}

// 16x16 tiles.  A warp covers one 16-row tile row and eight consecutive
// blocks: lane l handles row l % 16 and the four consecutive blocks
// 4 (l / 16) .. 4 (l / 16) + 3 (128 contiguous bytes, all loads in flight
// together).  Each block's tile amax is a max over the 16 lanes of a
// half-warp (four shuffles); a lane's four scale bytes form one word.
template <bool RHT>
__global__ void __launch_bounds__(256) quant_nvfp4_2d_kernel(
    const uint16_t *__restrict__ x, int64_t M, int64_t K, int64_t ldx, uint32_t mask, const float *scale_src,
    int src_is_amax, float *gs_out, int write_gs, uint8_t *__restrict__ codes, uint8_t *__restrict__ sf) {
    grid_dependency_wait();
    grid_dependents_launch();
    __shared__ float den_tab[128], rcp_tab[128];
    const float s_g = src_is_amax ? global_scale_of(*scale_src) : *scale_src;
    if (write_gs && blockIdx.x == 0 && threadIdx.x == 0) *gs_out = s_g;
    const NvScale c = nv_scale_setup(s_g, den_tab, rcp_tab);
    uint32_t sw[8];
    rht_sign_words(mask, sw);
    const int64_t KB = K >> 4;
    const int64_t k8 = (KB + 7) >> 3;                 // groups of eight blocks per row
    const int64_t tasks = (M >> 4) * k8;
    const bool pack4 = (KB & 3) == 0;
    const int lane = threadIdx.x & 31;
    const int r16 = lane & 15, hw = lane >> 4;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t task = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); task < tasks; task += warps) {
        const int64_t rt = task / k8, g8 = task - rt * k8;
        const int64_t row = rt * 16 + r16;
        const int64_t kb0 = g8 * 8 + 4 * hw;
        const uint16_t *rp = x + row * ldx;
        uint32_t w[4][8];
#pragma unroll
        for (int i = 0; i < 4; i++) load_words16(rp + (kb0 + i < KB ? kb0 + i : 0) * 16, w[i]);
        uint32_t sbw = 0;
        uint2 cd[4];
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const bool v = kb0 + i < KB;  // uniform over the half-warp
            f32x2 P[8];
            if (RHT) rht16_u_words(w[i], sw, P);
            else words_to_pairs(w[i], P);
            float mu = v ? pairs_absmax3(P) : 0.0f;
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) mu = fmaxf(mu, __shfl_xor_sync(0xFFFFFFFFu, mu, o));
            const float tmax = RHT ? __fmul_rn(mu, 0.25f) : mu;
            const uint32_t sb = nv_scale_code(tmax, 6.0f, c.c6, c);
            sbw |= (sb & 0xFFu) << (8 * i);
            cd[i] = sb ? nv_codes<RHT>(P, rcp_tab[sb], c.fast) : make_uint2(0u, 0u);
        }
        uint8_t *cp = codes + row * (K >> 1) + kb0 * 8;
        if (kb0 + 3 < KB && ((K >> 1) & 15) == 0) {  // 16-byte aligned: rows of a multiple of 32 codes bytes
            reinterpret_cast<uint4 *>(cp)[0] = make_uint4(cd[0].x, cd[0].y, cd[1].x, cd[1].y);
            reinterpret_cast<uint4 *>(cp)[1] = make_uint4(cd[2].x, cd[2].y, cd[3].x, cd[3].y);
        } else {
#pragma unroll
            for (int i = 0; i < 4; i++)
                if (kb0 + i < KB) reinterpret_cast<uint2 *>(cp)[i] = cd[i];
        }
        if (pack4) {
            if (kb0 < KB) *reinterpret_cast<uint32_t *>(sf + sf_word_offset(row, kb0 >> 2, KB)) = sbw;
        } else {
#pragma unroll
            for (int i = 0; i < 4; i++)
                if (kb0 + i < KB) sf[sf_offset(row, kb0 + i, KB)] = (uint8_t)(sbw >> (8 * i));
        }
    }
}

// ===================================================================== fused NVFP4
// One cooperative kernel per 16x16-block tensor (contiguous, no gather):
//   phase 1  amax over the tensor (four blocks per thread in flight);
//   barrier  every CTA arrives on a grid counter and waits (bounded);
//   phase 2  every CTA reads the amax, derives s_g and quantizes its tiles
//            in the reverse of the phase-1 order, so the most recently read
//            lines come from L2.
// The counter and the amax bits live in the first 8 bytes of the code
// buffer (zeroed by the caller).  Those bytes are the first tile's codes:
// their writer first waits until every CTA has arrived a second time, i.e.
// has read the amax.
BSQ_DEV unsigned int ld_acquire_gpu(const unsigned int *p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Thread 0 of the CTA waits (sleeping, bounded) until *ctr >= target.
BSQ_DEV bool wait_counter(const unsigned int *ctr, unsigned int target, unsigned int *err, unsigned int site) {
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_gpu(ctr) < target) {
        __nanosleep(100);
        if (globaltimer_ns() - t0 > 2000000000ull) {
            report_timeout(err, site);
            return false;
        }
    }
    return true;
}

// All CTAs of a cooperative launch: arrive once, wait for every CTA.
BSQ_DEV bool grid_barrier(unsigned int *ctr, unsigned int target, unsigned int *err, unsigned int site) {
    __shared__ int ok_sh;
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(ctr, 1u);
        ok_sh = wait_counter(ctr, target, err, site);
        __threadfence();
    }
    __syncthreads();
    return ok_sh != 0;
}

template <bool RHT>
__global__ void __launch_bounds__(256) quant_nvfp4_fused_kernel(
    const uint16_t *__restrict__ x, int64_t M, int64_t K, uint32_t mask, unsigned int *scratch,
    float *gs_out, uint8_t *__restrict__ codes, uint8_t *__restrict__ sf, unsigned int *err) {
    __shared__ float den_tab[128], rcp_tab[128];
    uint32_t sw[8];
    rht_sign_words(mask, sw);
    const int64_t KB = K >> 4, nblk = M * KB;
    const int lane = threadIdx.x & 31;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    // ---- phase 1: amax
    {
        float m = 0.0f;
        for (int64_t b = tid; b < nblk; b += 4 * stride) {
            uint32_t w[4][8];
#pragma unroll
            for (int i = 0; i < 4; i++)
                if (b + i * stride < nblk) load_words16(x + (b + i * stride) * 16, w[i]);
#pragma unroll
            for (int i = 0; i < 4; i++)
                if (b + i * stride < nblk) m = fmaxf(m, block_absmax<RHT>(w[i], sw));
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        __shared__ float red[8];
        if (lane == 0) red[threadIdx.x >> 5] = m;
        __syncthreads();
        if (threadIdx.x == 0) {
            float b = red[0];
            for (int i = 1; i < 8; i++) b = fmaxf(b, red[i]);
            atomicMax(scratch + 1, __float_as_uint(b));
        }
    }
    if (!grid_barrier(scratch, gridDim.x, err, 20)) return;
    const float amax = __uint_as_float(ld_acquire_gpu(scratch + 1));
    __syncthreads();
    if (threadIdx.x == 0) atomicAdd(scratch, 1u);  // this CTA has read the amax
    const float s_g = global_scale_of(amax);
    if (blockIdx.x == 0 && threadIdx.x == 0) *gs_out = s_g;
    const NvScale c = nv_scale_setup(s_g, den_tab, rcp_tab);
    const unsigned int all_read = 2u * gridDim.x;
    {
        // ---- phase 2, 16x16 tiles (warp = 16 rows x 8 blocks), reverse task order
        const int64_t k8 = (KB + 7) >> 3;
        const int64_t tasks = (M >> 4) * k8;
        const bool pack4 = (KB & 3) == 0;
        const int r16 = lane & 15, hw = lane >> 4;
        const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
        const int64_t wid = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
        const int64_t ntask = wid < tasks ? (tasks - 1 - wid) / warps + 1 : 0;
        for (int64_t j = ntask - 1; j >= 0; j--) {
            const int64_t task = wid + j * warps;
            const int64_t rt = task / k8, g8 = task - rt * k8;
            const int64_t row = rt * 16 + r16;
            const int64_t kb0 = g8 * 8 + 4 * hw;
            const uint16_t *rp = x + row * K;
            uint32_t w[4][8];
#pragma unroll
            for (int i = 0; i < 4; i++) load_words16(rp + (kb0 + i < KB ? kb0 + i : 0) * 16, w[i]);
            uint32_t sbw = 0;
            uint2 cd[4];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const bool v = kb0 + i < KB;
                f32x2 P[8];
                if (RHT) rht16_u_words(w[i], sw, P);
                else words_to_pairs(w[i], P);
                float mu = v ? pairs_absmax3(P) : 0.0f;
#pragma unroll
                for (int o = 1; o < 16; o <<= 1) mu = fmaxf(mu, __shfl_xor_sync(0xFFFFFFFFu, mu, o));
                const float tmax = RHT ? __fmul_rn(mu, 0.25f) : mu;
                const uint32_t sbb = nv_scale_code(tmax, 6.0f, c.c6, c);
                sbw |= (sbb & 0xFFu) << (8 * i);
                cd[i] = sbb ? nv_codes<RHT>(P, rcp_tab[sbb], c.fast) : make_uint2(0u, 0u);
            }
            if (task == 0) {  // holds the first block's codes: every CTA has read the amax
                if (lane == 0 && !wait_counter(scratch, all_read, err, 22)) cd[0] = make_uint2(0u, 0u);
                __syncwarp();
            }
            uint8_t *cp = codes + row * (K >> 1) + kb0 * 8;
            if (kb0 + 3 < KB && ((K >> 1) & 15) == 0) {
                reinterpret_cast<uint4 *>(cp)[0] = make_uint4(cd[0].x, cd[0].y, cd[1].x, cd[1].y);
                reinterpret_cast<uint4 *>(cp)[1] = make_uint4(cd[2].x, cd[2].y, cd[3].x, cd[3].y);
            } else {
#pragma unroll
                for (int i = 0; i < 4; i++)
                    if (kb0 + i < KB) reinterpret_cast<uint2 *>(cp)[i] = cd[i];
            }
            if (pack4) {
                if (kb0 < KB) *reinterpret_cast<uint32_t *>(sf + sf_word_offset(row, kb0 >> 2, KB)) = sbw;
            } else {
#pragma unroll
                for (int i = 0; i < 4; i++)
                    if (kb0 + i < KB) sf[sf_offset(row, kb0 + i, KB)] = (uint8_t)(sbw >> (8 * i));
            }
        }
    }
}

// Division by an invariant divisor d <= 2^31 for n < 2^32 (Granlund and
// Montgomery, PLDI 1994): with s = ceil(log2 d) and m = ceil(2^(32+s) / d),
// floor(n / d) = (n * m) >> (32 + s).  m < 2^33 is kept in 64 bits.
struct DivU32 {
    uint64_t m;
    int sh;
};
static DivU32 divu32_for(uint32_t d) {
    int s = 0;
    while ((uint64_t(1) << s) < d) s++;
    const unsigned __int128 num = (unsigned __int128)1 << (32 + s);
    return {(uint64_t)((num + d - 1) / d), 32 + s};
}
BSQ_DEV uint32_t divu32(uint32_t n, const DivU32 &dv) {
    return (uint32_t)(((unsigned __int128)n * dv.m) >> dv.sh);
}


// ===================================================================== streaming NVFP4 (bulk-copy ring)
// Contiguous tensors (ldx == K, K % 64 == 0).  A CTA is one producer warp
// and eight consumer warps.  The producer's lane 0 streams chunks of the
// tensor into a ring of shared-memory stages with cp.async.bulk (completion
// on the stage's "full" mbarrier); the consumers read a stage, release it
// (one arrive per warp on its "empty" mbarrier) and compute.  The loads run
// ahead of the arithmetic by the whole ring, so every SM keeps
// kStages * 16 KB in flight whatever the consumers are doing.
//   1x16:  chunk = 512 consecutive blocks of 16 (16 KB); consumer thread t
//          takes blocks t and t + 256.
//   16x16: chunk = 16 rows x 512 columns (16 row copies of 1 KB, staged at a
//          1040-byte row stride so that the reads below hit distinct banks);
//          consumer thread t takes row t % 16, blocks 2 (t / 16) and
//          2 (t / 16) + 1 of the chunk: a half-warp holds one tile column.
// Modes: AMAX (amax only, into *amax_bits; with a counter the last CTA
// also writes s_g),
// QUANT (s_g from a given amax or scale), FUSED (amax over every chunk, a
// grid barrier, then the quantization in reverse chunk order so the most
// recently read lines come from L2; cooperative launch).  Every wait is
// bounded; on expiry the error word is set, the CTA drains its own copies
// and returns.
namespace nvs {
constexpr int kConsumerWarps = 8;
constexpr int kThreads = 32 * (1 + kConsumerWarps);
constexpr int kStages = 4;
constexpr int kRowStride = 1040;                 // 16x16: bytes per staged row (1 KB + 16)
constexpr int kStageBytes = 16 * kRowStride;     // also holds a 16 KB 1x16 chunk
constexpr int kSmemBytes = kStages * kStageBytes;
constexpr uint64_t kTimeoutNs = 2000000000ull;
enum { AMAX = 0, QUANT = 1, FUSED = 2 };
}  // namespace nvs

// Consumer-only barrier (named barrier 1: the 256 consumer threads).
BSQ_DEV void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(32 * nvs::kConsumerWarps) : "memory"); }

// Chunk geometry.  1x16: chunk c covers flat blocks [512 c, 512 c + 512).
// 16x16: chunk c = (row group rg, span sp) covers rows 16 rg .. 16 rg + 15
// and columns 512 sp .. 512 sp + 511 (the last span may be shorter).
struct NvChunks {
    int64_t M, K, KB, nblk;
    int64_t nspan;   // 16x16: spans per row group
    int64_t count;
};

template <bool TWO_D>
BSQ_DEV NvChunks nv_chunks(int64_t M, int64_t K) {
    NvChunks g;
    g.M = M;
    g.K = K;
    g.KB = K >> 4;
    g.nblk = M * g.KB;
    g.nspan = (K + 511) >> 9;
    g.count = TWO_D ? (M >> 4) * g.nspan : (g.nblk + 511) >> 9;
    return g;
}

template <int MODE, bool RHT, bool TWO_D>
__global__ void __launch_bounds__(nvs::kThreads, 2) quant_nvfp4_stream_kernel(
    const uint16_t *__restrict__ x, int64_t M, int64_t K, DivU32 div_kb, DivU32 div_span, uint32_t mask,
    unsigned int *counter,
    unsigned int *amax_bits, const float *scale_src, int src_is_amax, float *gs_out, uint8_t *__restrict__ codes,
    uint8_t *__restrict__ sf, unsigned int *err) {
    using namespace sm100;
    grid_dependency_wait();
    grid_dependents_launch();
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ __align__(8) uint64_t full_bar[nvs::kStages], empty_bar[nvs::kStages];
    __shared__ float den_tab[128], rcp_tab[128];
    __shared__ float red[nvs::kConsumerWarps];
    __shared__ volatile int abort_flag;
    __shared__ int ok_sh;
    const NvChunks g = nv_chunks<TWO_D>(M, K);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // chunks of this CTA: c = blockIdx.x + i * gridDim.x, i < my (32-bit
    // counters: fewer than 2^32 chunks on this path)
    const uint32_t my = blockIdx.x < g.count ? (uint32_t)(g.count - 1 - blockIdx.x) / gridDim.x + 1 : 0u;
    const uint32_t total = (MODE == nvs::FUSED ? 2u : 1u) * my;  // stage fills in this CTA's sequence
    if (threadIdx.x == 0) {
        for (int i = 0; i < nvs::kStages; i++) {
            mbar_init(smem_u32(&full_bar[i]), 1);
            mbar_init(smem_u32(&empty_bar[i]), nvs::kConsumerWarps);
        }
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    // j-th fill of the sequence -> chunk index (FUSED: forward, then reverse)
    auto chunk_of = [&](uint32_t j) -> uint32_t {
        const uint32_t i = (MODE == nvs::FUSED && j >= my) ? (2 * my - 1 - j) : j;
        return blockIdx.x + i * gridDim.x;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        uint32_t armed = 0, armed_par = 0;
        for (uint32_t j = 0; j < total; j++) {
            const int s = (int)(j % nvs::kStages);
            const uint32_t ph = (uint32_t)((j / nvs::kStages) & 1);
            bool ok = true;
            if (lane == 0) ok = mbar_wait(smem_u32(&empty_bar[s]), ph ^ 1u, &abort_flag, err, 30, nvs::kTimeoutNs);
            if (!__shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0)) break;
            const int64_t c = chunk_of(j);
            uint8_t *dst = ring + s * nvs::kStageBytes;
            const uint32_t fb = smem_u32(&full_bar[s]);
            if (!TWO_D) {
                if (lane == 0) {
                    const int64_t b0 = c << 9;
                    const int64_t nb = (g.nblk - b0) < 512 ? (g.nblk - b0) : 512;
                    mbar_arrive_expect_tx(fb, (uint32_t)(nb * 32));
                    bulk_load(smem_u32(dst), x + b0 * 16, (uint32_t)(nb * 32), fb);
                }
            } else {
                // chunk counts stay below 2^32 on this path (stream_ok): 32-bit division
                const uint32_t rg = divu32((uint32_t)c, div_span), sp = (uint32_t)c - rg * (uint32_t)g.nspan;
                const int64_t k0 = (int64_t)sp << 9;
                const int64_t cols = (K - k0) < 512 ? (K - k0) : 512;
                if (lane == 0) mbar_arrive_expect_tx(fb, (uint32_t)(16 * cols * 2));
                __syncwarp();
                if (lane < 16)
                    bulk_load(smem_u32(dst + lane * nvs::kRowStride), x + (rg * 16 + lane) * K + k0,
                              (uint32_t)(cols * 2), fb);
            }
            armed |= 1u << s;
            armed_par = (armed_par & ~(1u << s)) | (ph << s);
        }
        // before exit every copy of this CTA has landed (normally the
        // consumers have already waited for all of them)
        if (lane == 0)
            for (int i = 0; i < nvs::kStages; i++)
                if (armed & (1u << i)) {
                    volatile int never = 0;
                    mbar_wait(smem_u32(&full_bar[i]), (armed_par >> i) & 1u, &never, err, 31, nvs::kTimeoutNs);
                }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int t = threadIdx.x - 32;  // 0..255
    uint32_t sw[8];
    rht_sign_words(mask, sw);
    uint32_t j = 0;
    // waits for fill j; false when the CTA gives up
    auto acquire = [&](uint32_t jj) -> const uint8_t * {
        const int s = (int)(jj % nvs::kStages);
        const uint32_t ph = (uint32_t)((jj / nvs::kStages) & 1);
        const bool ok = mbar_wait(smem_u32(&full_bar[s]), ph, &abort_flag, err, 32, nvs::kTimeoutNs);
        if (!__all_sync(0xFFFFFFFFu, ok)) return nullptr;
        return ring + s * nvs::kStageBytes;
    };
    auto release = [&](uint32_t jj) {
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty_bar[jj % nvs::kStages]));
    };
    // the 8 words of 1x16 block `slot` (0..511) of a staged chunk; the two
    // 16-byte halves are read in an order that spreads each quarter-warp
    // over all 32 banks
    auto words_1d = [&](const uint8_t *st, int slot, uint32_t w[8]) {
        const int h = (slot >> 2) & 1;
        const uint4 a = *reinterpret_cast<const uint4 *>(st + slot * 32 + 16 * h);
        const uint4 b = *reinterpret_cast<const uint4 *>(st + slot * 32 + 16 * (h ^ 1));
        const uint4 lo = h ? b : a, hi = h ? a : b;
        w[0] = lo.x; w[1] = lo.y; w[2] = lo.z; w[3] = lo.w;
        w[4] = hi.x; w[5] = hi.y; w[6] = hi.z; w[7] = hi.w;
    };
    auto words_2d = [&](const uint8_t *st, int row, int blk, uint32_t w[8]) {
        const uint4 a = *reinterpret_cast<const uint4 *>(st + row * nvs::kRowStride + blk * 32);
        const uint4 b = *reinterpret_cast<const uint4 *>(st + row * nvs::kRowStride + blk * 32 + 16);
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
        w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    };

    // A wait that gives up sets the CTA's abort flag; the consumer warps then
    // skip the rest of the work but still pass every named barrier below.
    bool alive = true;
    float s_g = 1.0f;
    if (MODE != nvs::QUANT) {
        // ---- amax over this CTA's chunks
        float m = 0.0f;
        for (; j < my && alive; j++) {
            const uint8_t *st = acquire(j);
            if (!st) {
                alive = false;
                break;
            }
            const int64_t c = chunk_of(j);
            if (!TWO_D) {
                const int64_t nb = g.nblk - (c << 9);
                uint32_t w0[8], w1[8];
                if (t < nb) words_1d(st, t, w0);
                if (t + 256 < nb) words_1d(st, t + 256, w1);
                release(j);
                if (t < nb) m = fmaxf(m, block_absmax<RHT>(w0, sw));
                if (t + 256 < nb) m = fmaxf(m, block_absmax<RHT>(w1, sw));
            } else {
                const uint32_t sp = (uint32_t)c - divu32((uint32_t)c, div_span) * (uint32_t)g.nspan;
                const int64_t nb = (K - (sp << 9)) >> 4;
                const int row = t & 15, b0 = 2 * (t >> 4);
                uint32_t w0[8], w1[8];
                if (b0 < nb) words_2d(st, row, b0, w0);
                if (b0 + 1 < nb) words_2d(st, row, b0 + 1, w1);
                release(j);
                if (b0 < nb) m = fmaxf(m, block_absmax<RHT>(w0, sw));
                if (b0 + 1 < nb) m = fmaxf(m, block_absmax<RHT>(w1, sw));
            }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (lane == 0) red[warp - 1] = m;
        consumers_sync();
        if (t == 0) {
            ok_sh = 0;
            if (!abort_flag) {
                float b = red[0];
                for (int i = 1; i < nvs::kConsumerWarps; i++) b = fmaxf(b, red[i]);
                atomicMax(amax_bits, __float_as_uint(b));
                __threadfence();
                if (MODE == nvs::AMAX) {
                    // with a counter, the last CTA turns the amax into s_g
                    if (counter && atomicAdd(counter, 1u) == gridDim.x - 1) {
                        __threadfence();
                        *gs_out = global_scale_of(__uint_as_float(atomicOr(amax_bits, 0u)));
                    }
                } else {
                    atomicAdd(counter, 1u);
                    ok_sh = wait_counter(counter, gridDim.x, err, 33);
                    if (!ok_sh) abort_flag = 1;   // the producer stops too
                }
            }
        }
        if (MODE == nvs::AMAX) return;
        consumers_sync();
        if (ok_sh) {
            s_g = global_scale_of(__uint_as_float(ld_acquire_gpu(amax_bits)));
        } else {
            alive = false;
        }
        consumers_sync();
        if (t == 0 && alive) atomicAdd(counter, 1u);  // this CTA has read the amax
        if (alive && blockIdx.x == 0 && t == 0) *gs_out = s_g;
    } else {
        s_g = src_is_amax ? global_scale_of(*scale_src) : *scale_src;
        if (gs_out && blockIdx.x == 0 && t == 0) *gs_out = s_g;
    }
    // den / rcp tables (threads 0..127 of the consumers)
    if (t < 128) {
        const float den = __fmul_rn(e4m3_to_f32(t), s_g);
        den_tab[t] = den;
        rcp_tab[t] = (t == 0 || t == 127) ? 0.0f : __frcp_rn(den);
    }
    consumers_sync();
    NvScale cs;
    cs.s_g = s_g;
    cs.c6 = __frcp_rn(__fmul_rn(6.0f, s_g));
    cs.c4 = __frcp_rn(__fmul_rn(4.0f, s_g));
    cs.fast = s_g >= 0x1p-90f && s_g <= 0x1p100f;
    const unsigned int all_read = 2u * gridDim.x;

    // ---- quantize this CTA's chunks (FUSED: in reverse order)
    const uint32_t jend = (MODE == nvs::FUSED) ? 2 * my : my;
    for (; j < jend && alive; j++) {
        const uint8_t *st = acquire(j);
        if (!st) break;
        const int64_t c = chunk_of(j);
        if (!TWO_D) {
            // 32-bit block indices (M * K / 16 < 2^32 on this path)
            const uint32_t b0 = (uint32_t)c << 9;
            const int64_t nb = g.nblk - (int64_t)b0;
            const uint32_t kb32 = (uint32_t)g.KB, bt = (kb32 + 3) >> 2;
            uint32_t w0[8], w1[8];
            words_1d(st, t, w0);   // slots past the tensor's end hold stale bytes: never stored
            words_1d(st, t + 256, w1);
            release(j);
#pragma unroll
            for (int h = 0; h < 2; h++) {
                const int slot = t + 256 * h;
                const bool v = slot < nb;
                const uint32_t b = b0 + slot;
                uint32_t sb;
                uint2 cd;
                nv_block_1d<RHT, false>(h ? w1 : w0, sw, cs, den_tab, rcp_tab, sb, cd);
                // the first block's codes double as the amax scratch: written
                // once every CTA has read the amax
                if (MODE == nvs::FUSED && v && b == 0 && !wait_counter(counter, all_read, err, 34))
                    cd = make_uint2(0u, 0u);
                if (v) *reinterpret_cast<uint2 *>(codes + (size_t)b * 8) = cd;
                // lanes 4j..4j+3 hold blocks 4i..4i+3 of one row (K % 64 == 0):
                // one scale word at the swizzled offset of (row, 4-block group)
                const uint32_t b1 = __shfl_down_sync(0xFFFFFFFFu, sb, 1);
                const uint32_t b2 = __shfl_down_sync(0xFFFFFFFFu, sb, 2);
                const uint32_t b3 = __shfl_down_sync(0xFFFFFFFFu, sb, 3);
                if (v && (lane & 3) == 0) {
                    const uint32_t r = divu32(b, div_kb), b4 = (b - r * kb32) >> 2;
                    const uint32_t off = (((r >> 7) * bt + b4) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2);
                    *reinterpret_cast<uint32_t *>(sf + off) =
                        (sb & 0xFFu) | ((b1 & 0xFFu) << 8) | ((b2 & 0xFFu) << 16) | ((b3 & 0xFFu) << 24);
                }
            }
        } else {
            // 32-bit chunk, row and block indices (M * K / 16 < 2^32 on this path)
            const uint32_t rg = divu32((uint32_t)c, div_span), sp = (uint32_t)c - rg * (uint32_t)g.nspan;
            const int64_t nb = (K - ((int64_t)sp << 9)) >> 4;  // blocks in this span (multiple of 4)
            const int row = t & 15, bp = t >> 4;
            const uint32_t grow = rg * 16 + row;
            const uint32_t kb0 = (sp << 5) + 2 * bp;          // first block of this thread
            const bool v = 2 * bp < nb;                    // both blocks valid (nb is even)
            uint32_t w[2][8];
            words_2d(st, row, v ? 2 * bp : 0, w[0]);
            words_2d(st, row, v ? 2 * bp + 1 : 0, w[1]);
            release(j);
            uint2 cd[2];
            uint32_t sbw = 0;
#pragma unroll
            for (int i = 0; i < 2; i++) {
                f32x2 P[8];
                if (RHT) rht16_u_words(w[i], sw, P);
                else words_to_pairs(w[i], P);
                float mu = v ? pairs_absmax3(P) : 0.0f;
#pragma unroll
                for (int o = 1; o < 16; o <<= 1) mu = fmaxf(mu, __shfl_xor_sync(0xFFFFFFFFu, mu, o));
                const float tmax = RHT ? __fmul_rn(mu, 0.25f) : mu;
                const uint32_t sb = nv_scale_code(tmax, 6.0f, cs.c6, cs);
                sbw |= (sb & 0xFFu) << (8 * i);
                cd[i] = sb ? nv_codes<RHT>(P, rcp_tab[sb], cs.fast) : make_uint2(0u, 0u);
            }
            if (MODE == nvs::FUSED && v && grow == 0 && kb0 == 0 && !wait_counter(counter, all_read, err, 35))
                cd[0] = make_uint2(0u, 0u);
            if (v)
                *reinterpret_cast<uint4 *>(codes + (size_t)grow * (uint32_t)(K >> 1) + kb0 * 8) =
                    make_uint4(cd[0].x, cd[0].y, cd[1].x, cd[1].y);
            // lanes l and l + 16 hold blocks 4i .. 4i + 3 of one row: one word,
            // at the swizzled offset of (row, 4-block group) (sf_word_offset in
            // 32-bit arithmetic: the scale buffer holds fewer than 2^32 bytes)
            const uint32_t other = __shfl_down_sync(0xFFFFFFFFu, sbw, 16);
            if (v && lane < 16) {
                const uint32_t bt = (uint32_t)((g.KB + 3) >> 2);
                const uint32_t off = (((grow >> 7) * bt + (kb0 >> 2)) << 9) + ((grow & 31) << 4) + (((grow >> 5) & 3) << 2);
                *reinterpret_cast<uint32_t *>(sf + off) = sbw | (other << 16);
            }
        }
    }
}

// ===================================================================== MXFP8
// E8M0 code of a block from its absolute maximum m >= 0, i.e.
// clamp(floor(log2 m) - 8, -127, 127) + 127.  The biased exponent field f of
// a normal m is floor(log2 m) + 127, so the code is f - 8; a subnormal or
// zero m (f = 0) takes the lower clamp, code 0; the largest finite field
// (254) gives 246, so the upper clamp never applies.
BSQ_DEV uint32_t mx_scale_code(float m) {
    const int f = (int)(__float_as_uint(m) >> 23);
    return (uint32_t)max(f - 8, 0);
}
// 2^-E for the block exponent E = code - 127, as the binary32 with exponent
// field 254 - code (8..254: always normal).
BSQ_DEV float mx_inv_scale(uint32_t code) { return __uint_as_float((254u - code) << 23); }

// s = v * 2^-E for 8 values (exact: a power of two, no overflow), on fp32
// pairs.
BSQ_DEV void mx_scale8(const float v[8], float inv, float s[8]) {
    const f32x2 I = f2_pack(inv, inv);
#pragma unroll
    for (int k = 0; k < 4; k++) f2_unpack(f2_mul(f2_pack(v[2 * k], v[2 * k + 1]), I), s[2 * k], s[2 * k + 1]);
}

// RNE of 8 scaled values to E4M3, element 0 in the lowest byte.  The
// satfinite conversion returns +-448 for |s| > 448, which is what clamping
// to +-448 first and then rounding gives.
BSQ_DEV uint2 mx_rne8(const float s[8]) {
    uint2 r;
    asm("{\n\t.reg .b16 h0, h1, h2, h3;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 h0, %3, %2;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 h1, %5, %4;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 h2, %7, %6;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 h3, %9, %8;\n\t"
        "mov.b32 %0, {h0, h1};\n\t"
        "mov.b32 %1, {h2, h3};\n\t}"
        : "=r"(r.x), "=r"(r.y)
        : "f"(s[0]), "f"(s[1]), "f"(s[2]), "f"(s[3]), "f"(s[4]), "f"(s[5]), "f"(s[6]), "f"(s[7]));
    return r;
}

// Stochastic rounding of 8 scaled values to E4M3 with the four words of one
// Philox call: element i draws the low (even i) or high (odd i) 16 bits of
// word i/2.  Integer form of e4m3_sr for 2^-6 <= a <= 448, a = min(|s|, 448)
// (a's bits are read as an unsigned integer): the E4M3 neighbour below a is
// a with its low 20 bits cleared and frac = low20(a) / 2^20, so rounding up
// happens iff 16 r16 < low20(a).  Shifted left by 4 and with the exponent
// rebias 120 << 23 taken out, t = (a << 4) + 0xFFFFF0 - (r16 << 8) - (120 << 27)
// (mod 2^32) carries into bit 24 exactly when rounding up, and its top byte
// is then the code's magnitude (E4M3 exponent and three mantissa bits; bit 31
// stays clear since a <= 448).  r16 << 8 is one byte permute of the draw
// word.  A chunk holding some a < 2^-6 (E4M3 subnormals, zeros) runs the
// float form for all eight values.
// The float form of stochastic rounding for a whole chunk (e4m3_sr per value
// after the clamp to +-448).  It runs only for chunks holding E4M3 subnormals
// or zeros, so it is kept out of line: the unrolled callers stay small.
__device__ __noinline__ uint2 mx_sr8_float(float s0, float s1, float s2, float s3, float s4, float s5, float s6,
                                           float s7, uint4 rnd) {
    const float s[8] = {s0, s1, s2, s3, s4, s5, s6, s7};
    const uint32_t w[4] = {rnd.x, rnd.y, rnd.z, rnd.w};
    uint32_t c[8];
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const float v = fminf(fmaxf(s[i], -448.0f), 448.0f);
        c[i] = e4m3_sr(v, (i & 1) ? (w[i >> 1] >> 16) : (w[i >> 1] & 0xFFFFu));
    }
    return make_uint2(c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24), c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24));
}

// The same with zeros allowed (a zero never rounds: its code is the sign);
// the float form runs only when some nonzero value lies below 2^-6.  Inline
// for inputs where zeros are common (decoded 4-bit data), and out of line as
// the fallback of mx_sr8.
BSQ_DEV uint2 mx_sr8_z(const float s[8], uint4 rnd) {
    const uint32_t w[4] = {rnd.x, rnd.y, rnd.z, rnd.w};
    uint32_t b[8];
    bool slow = false;
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const uint32_t a = __float_as_uint(fminf(fabsf(s[i]), 448.0f));
        slow |= a - 1u < 0x3C7FFFFFu;  // 0 < a < 2^-6
        const uint32_t p = __byte_perm(w[i >> 1], 0u, (i & 1) ? 0x4324u : 0x4104u);
        const uint32_t t = (a << 4) + 0x40FFFFF0u - p;
        b[i] = (a ? t : 0u) | (__float_as_uint(s[i]) & 0x80000000u);
    }
    if (slow) return mx_sr8_float(s[0], s[1], s[2], s[3], s[4], s[5], s[6], s[7], rnd);
    return make_uint2(__byte_perm(__byte_perm(b[0], b[1], 0x0073u), __byte_perm(b[2], b[3], 0x7300u), 0x7610u),
                      __byte_perm(__byte_perm(b[4], b[5], 0x0073u), __byte_perm(b[6], b[7], 0x7300u), 0x7610u));
}
__device__ __noinline__ uint2 mx_sr8_zeros(float s0, float s1, float s2, float s3, float s4, float s5, float s6,
                                           float s7, uint4 rnd) {
    const float s[8] = {s0, s1, s2, s3, s4, s5, s6, s7};
    return mx_sr8_z(s, rnd);
}

BSQ_DEV uint2 mx_sr8(const float s[8], uint4 rnd) {
    const uint32_t w[4] = {rnd.x, rnd.y, rnd.z, rnd.w};
    uint32_t b[8];
    bool slow = false;
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const uint32_t a = __float_as_uint(fminf(fabsf(s[i]), 448.0f));
        slow |= a < 0x3C800000u;  // 2^-6
        const uint32_t p = __byte_perm(w[i >> 1], 0u, (i & 1) ? 0x4324u : 0x4104u);  // r16 << 8
        const uint32_t t = (a << 4) + 0x40FFFFF0u - p;  // 0xFFFFF0 - (120 << 27) mod 2^32
        b[i] = t | (__float_as_uint(s[i]) & 0x80000000u);
    }
    if (slow) return mx_sr8_zeros(s[0], s[1], s[2], s[3], s[4], s[5], s[6], s[7], rnd);
    return make_uint2(__byte_perm(__byte_perm(b[0], b[1], 0x0073u), __byte_perm(b[2], b[3], 0x7300u), 0x7610u),
                      __byte_perm(__byte_perm(b[4], b[5], 0x0073u), __byte_perm(b[6], b[7], 0x7300u), 0x7610u));
}

BSQ_DEV uint4 mx_draws(uint64_t chunk, const PhiloxKeys &keys, uint32_t stream_id) {
    return philox4x32_10(make_uint4((uint32_t)chunk, (uint32_t)(chunk >> 32), stream_id, 0u), keys);
}

// True when stochastic rounding of the 8 scaled values cannot depend on the
// draws: each one is zero or an E4M3 value of the normal range or above 448
// (its low 20 bits are zero, so frac = 0 and it never rounds up), as every
// E4M3 input rescaled by a power of two is unless it falls below 2^-6.  Such
// a chunk's codes are its nearest-even codes (exact values, saturated above
// 448 as stochastic rounding saturates them).
BSQ_DEV bool mx_sr8_drawless(const float s[8]) {
    bool ok = true;
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const uint32_t a = __float_as_uint(fminf(fabsf(s[i]), 448.0f));
        ok &= ((a & 0xFFFFFu) == 0u) & ((a >= 0x3C800000u) | (a == 0u));
    }
    return ok;
}

// Philox draws and rounding of one chunk, out of line (the rare case of the
// EXACT_IN path below).
__device__ __noinline__ uint2 mx_sr8_drawn(float s0, float s1, float s2, float s3, float s4, float s5, float s6,
                                           float s7, uint64_t chunk, const PhiloxKeys &keys,
                                           uint32_t stream_id) {
    const float s[8] = {s0, s1, s2, s3, s4, s5, s6, s7};
    return mx_sr8(s, mx_draws(chunk, keys, stream_id));
}

// The 8 codes of one chunk of a block with E8M0 code sb (zero: the block's
// maximum is 0, whose codes are all +0).  chunk is the output linear index
// of the chunk's first element divided by 8: the Philox counter of SR.  With
// EXACT_IN (inputs that are E4M3 values times a power of two) the Philox call
// runs only for chunks whose rounding can depend on it.
template <bool SR, bool EXACT_IN = false, bool ZEROS = false>
BSQ_DEV uint2 mx_encode8(const float v[8], bool zero, uint32_t sb, uint64_t chunk, const PhiloxKeys &keys,
                         uint32_t stream_id) {
    float s[8];
    mx_scale8(v, mx_inv_scale(sb), s);
    uint2 q;
    if (SR) {
        if (ZEROS)
            q = mx_sr8_z(s, mx_draws(chunk, keys, stream_id));
        else if (!EXACT_IN)
            q = mx_sr8(s, mx_draws(chunk, keys, stream_id));
        else if (mx_sr8_drawless(s))
            q = mx_rne8(s);
        else
            q = mx_sr8_drawn(s[0], s[1], s[2], s[3], s[4], s[5], s[6], s[7], chunk, keys, stream_id);
    } else {
        q = mx_rne8(s);
    }
    return zero ? make_uint2(0u, 0u) : q;
}

// ---- MXFP8 stochastic rounding on packed bf16 pairs (16-bit lanes)
BSQ_DEV uint32_t u16x2_max(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
BSQ_DEV uint32_t u16x2_min(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("min.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
BSQ_DEV uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// |x| bits of a chunk held as 4 bf16 pairs (element 2k in the low half of
// pair k) and the chunk's absolute maximum as bf16 bits (non-negative
// floats order as their bit patterns).
BSQ_DEV uint32_t bf16_chunk_absmax(const uint32_t p[4], uint32_t a[4]) {
#pragma unroll
    for (int k = 0; k < 4; k++) a[k] = p[k] & 0x7FFF7FFFu;
    const uint32_t m2 = u16x2_max(u16x2_max(a[0], a[1]), u16x2_max(a[2], a[3]));
    return max(m2 & 0xFFFFu, m2 >> 16);
}
// E8M0 code from a block maximum given as bf16 bits (exponent field in bits
// 7..14, the same field as the fp32 value's): see mx_scale_code.
BSQ_DEV uint32_t mx_scale_code_bf16(uint32_t m) { return (uint32_t)max((int)(m >> 7) - 8, 0); }

// Stochastic rounding of one chunk of bf16 values (pairs p, magnitudes a)
// in block code sb, two values per 32-bit operation.  s = |x| 2^-E is one
// bf16 multiply (exact whenever s >= 2^-126), clamped to 448 (0x43E0).  A
// bf16-sourced s has 4 bits below the E4M3 mantissa, so frac = low4 / 16 and
// "16 r16 < low20" becomes "r16 >> 12 < low4": adding 15 - (r16 >> 12) to
// the 16-bit lane carries into bit 4 exactly when rounding up, and
// (s + 15 - (r16 >> 12) - (120 << 7)) >> 4 is then the E4M3 magnitude code
// (exponent - 120 and three mantissa bits).  Shifted left by 4, each lane's
// code sits in its upper byte with bit 7 clear, where the bf16 sign bit is
// or-ed in.  A chunk holding some s < 2^-6 is redone with zeros allowed: a
// zero input lane (which never rounds) is computed as s = 2^-6 so that no
// borrow crosses into the other lane, and its code masked to the sign; only
// a chunk with some nonzero input below 2^-6 (E4M3 subnormals, or a product
// that underflowed) runs the fp32 form on all eight values.
// The fallback of mx_sr8_bf16 for a chunk that failed its fast check (out of
// line: the unrolled callers stay small).
__device__ __noinline__ uint2 mx_sr8_bf16_slow(uint4 pv, uint4 av, uint32_t sb, uint4 rnd) {
    const uint32_t p[4] = {pv.x, pv.y, pv.z, pv.w}, a[4] = {av.x, av.y, av.z, av.w};
    const uint32_t inv2 = ((254u - sb) << 7) * 0x10001u;
    const uint32_t w[4] = {rnd.x, rnd.y, rnd.z, rnd.w};
    uint32_t mn = 0xFFFFFFFFu, u[4];
#pragma unroll
    for (int k = 0; k < 4; k++) {
        const uint32_t s0 = u16x2_min(bf16x2_mul(a[k], inv2), 0x43E043E0u);
        const uint32_t nz = __vcmpne2(a[k], 0u);         // 0xFFFF in each nonzero input lane
        const uint32_t s = s0 | (~nz & 0x3C803C80u);
        mn = u16x2_min(mn, s);
        const uint32_t r = (~w[k] >> 12) & 0x000F000Fu;
        u[k] = (((s + r - 0x3C003C00u) << 4) & nz) | (p[k] & 0x80008000u);
    }
    if (min(mn & 0xFFFFu, mn >> 16) < 0x3C80u) {
        float v[8], sc[8];
#pragma unroll
        for (int k = 0; k < 4; k++) {
            v[2 * k] = bf16_lo(p[k]);
            v[2 * k + 1] = bf16_hi(p[k]);
        }
        mx_scale8(v, mx_inv_scale(sb), sc);
        return mx_sr8_float(sc[0], sc[1], sc[2], sc[3], sc[4], sc[5], sc[6], sc[7], rnd);
    }
    return make_uint2(__byte_perm(u[0], u[1], 0x7531u), __byte_perm(u[2], u[3], 0x7531u));
}

BSQ_DEV uint2 mx_sr8_bf16(const uint32_t p[4], const uint32_t a[4], uint32_t sb, uint4 rnd) {
    const uint32_t inv2 = ((254u - sb) << 7) * 0x10001u;  // 2^-E in both bf16 lanes
    const uint32_t w[4] = {rnd.x, rnd.y, rnd.z, rnd.w};
    uint32_t mn = 0xFFFFFFFFu, u[4];
#pragma unroll
    for (int k = 0; k < 4; k++) {
        const uint32_t s = u16x2_min(bf16x2_mul(a[k], inv2), 0x43E043E0u);
        mn = u16x2_min(mn, s);
        const uint32_t r = (~w[k] >> 12) & 0x000F000Fu;  // 15 - (r16 >> 12), both lanes
        u[k] = ((s + r - 0x3C003C00u) << 4) | (p[k] & 0x80008000u);
    }
    if (min(mn & 0xFFFFu, mn >> 16) < 0x3C80u)  // 2^-6
        return mx_sr8_bf16_slow(make_uint4(p[0], p[1], p[2], p[3]), make_uint4(a[0], a[1], a[2], a[3]), sb, rnd);
    return make_uint2(__byte_perm(u[0], u[1], 0x7531u), __byte_perm(u[2], u[3], 0x7531u));
}
// Row-wise: one thread per 8 elements, 4 lanes per block of 32.
// I: the index type of the per-chunk offsets and Philox counters (uint32_t
// when M * ldx < 2^31: single 32-bit instructions).
template <bool SR, typename I>
__global__ void __launch_bounds__(256) quant_mxfp8_row_kernel(
    const uint16_t *__restrict__ x, int64_t M, int64_t K, int64_t ldx, const __grid_constant__ PhiloxKeys keys,
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
            load8_bf16(x + (size_t)((I)rr * (I)ldx + (I)cc * 8), v);
            float m = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; i++) m = fmaxf(m, fabsf(v[i]));
            m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
            m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
            const bool zero = (m == 0.0f);
            const uint32_t sb = mx_scale_code(m);
            const I o = (I)rr * (I)K + (I)cc * 8;  // output offset of this chunk
            const uint64_t chunk = (uint64_t)(o >> 3);
            uint2 q = mx_encode8<SR>(v, zero, sb, chunk, keys, stream_id);
            if (valid) *reinterpret_cast<uint2 *>(codes + (size_t)o) = q;
            // scale byte: lanes 4j hold block j; 4 blocks (16 lanes) per word
            const int64_t kb = cc >> 2;
            if (pack4) {
                uint32_t b1 = __shfl_down_sync(0xFFFFFFFFu, sb, 4);
                uint32_t b2 = __shfl_down_sync(0xFFFFFFFFu, sb, 8);
                uint32_t b3 = __shfl_down_sync(0xFFFFFFFFu, sb, 12);
                if (valid && (lane & 15) == 0)
                    *reinterpret_cast<uint32_t *>(sf + (size_t)sf_word_offset_t<I>((I)rr, (I)(kb >> 2), (I)KB)) =
                        sb | (b1 << 8) | (b2 << 16) | (b3 << 24);
            } else if (valid && (lane & 3) == 0) {
                sf[(size_t)sf_offset_t<I>((I)rr, (I)kb, (I)KB)] = (uint8_t)sb;
            }
        }
    }
}

// Row-wise for a contiguous tensor whose rows hold a multiple of 128
// elements: a flat sequence of 8-element chunks, four per thread in flight.
// Lanes 4j..4j+3 hold one block of 32 (two-step shuffle max); lanes 16i hold
// the first of four consecutive blocks of one row and store their scale
// word.  The SR draw index of a chunk is its flat position (row * K + col).
template <bool SR>
__global__ void __launch_bounds__(256) quant_mxfp8_row_flat_kernel(
    const uint16_t *__restrict__ x, int64_t nchunk, int64_t K, DivU32 div_k8, const __grid_constant__ PhiloxKeys keys,
    uint32_t stream_id, uint8_t *__restrict__ codes, uint8_t *__restrict__ sf) {
    constexpr int U = 4;
    const int64_t K8 = K >> 3, KB = K >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t nwarp = (nchunk + 31) & ~int64_t(31);
    for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c - lane < nwarp; c += U * stride) {
        uint4 raw[U];
#pragma unroll
        for (int h = 0; h < U; h++) {
            const int64_t cc = c + h * stride;
            raw[h] = __ldg(reinterpret_cast<const uint4 *>(x + (cc < nchunk ? cc : 0) * 8));
        }
#pragma unroll
        for (int h = 0; h < U; h++) {
            const int64_t cc = c + h * stride;
            const bool valid = cc < nchunk;
            if (h && !__any_sync(0xFFFFFFFFu, valid)) break;
            const uint32_t w[4] = {raw[h].x, raw[h].y, raw[h].z, raw[h].w};
            float v[8];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                v[2 * i] = bf16_lo(w[i]);
                v[2 * i + 1] = bf16_hi(w[i]);
            }
            float m = fmax3(fmax3(fabsf(v[0]), fabsf(v[1]), fabsf(v[2])), fmax3(fabsf(v[3]), fabsf(v[4]), fabsf(v[5])),
                            fmaxf(fabsf(v[6]), fabsf(v[7])));
            m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
            m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
            const bool zero = (m == 0.0f);
            const uint32_t sb = mx_scale_code(m);
            const uint2 q = mx_encode8<SR>(v, zero, sb, (uint64_t)cc, keys, stream_id);
            if (valid) *reinterpret_cast<uint2 *>(codes + cc * 8) = q;
            const uint32_t b1 = __shfl_down_sync(0xFFFFFFFFu, sb, 4);
            const uint32_t b2 = __shfl_down_sync(0xFFFFFFFFu, sb, 8);
            const uint32_t b3 = __shfl_down_sync(0xFFFFFFFFu, sb, 12);
            if (valid && (lane & 15) == 0) {
                const int64_t row = divu32((uint32_t)cc, div_k8), kb = (cc - row * K8) >> 2;
                *reinterpret_cast<uint32_t *>(sf + sf_word_offset(row, kb >> 2, KB)) =
                    sb | (b1 << 8) | (b2 << 16) | (b3 << 24);
            }
        }
    }
}

// Row-wise for a contiguous tensor whose rows hold a multiple of 1024
// elements.  A warp takes spans of 1024 consecutive elements (one row
// segment); lane l loads the 8-element chunks l, l+32, l+64, l+96 of the span
// (four 16-byte loads in flight, each warp-wide load reading 512 contiguous
// bytes).  Lanes 4j..4j+3 of a 32-chunk group hold one block of 32 (two-step
// shuffle max) and lane 4j stores its scale byte.  The SR draw index of a
// chunk is its flat position.
template <bool SR>
__global__ void __launch_bounds__(256) quant_mxfp8_row_span_kernel(
    const uint16_t *__restrict__ x, uint32_t nspan, int64_t K, DivU32 div_spr, const __grid_constant__ PhiloxKeys keys,
    uint32_t stream_id, uint8_t *__restrict__ codes, uint8_t *__restrict__ sf) {
    const int lane = threadIdx.x & 31;
    const uint32_t spr = (uint32_t)(K >> 10);  // spans per row
    const int64_t KB = K >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    const bool sf_lane = (lane & 3) == 0;
    for (uint32_t sp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; sp < nspan; sp += nwarps) {
        const int64_t e0 = (int64_t)sp << 10;
        const uint4 *src = reinterpret_cast<const uint4 *>(x + e0) + lane;
        uint4 raw[4];
#pragma unroll
        for (int h = 0; h < 4; h++) raw[h] = __ldg(src + 32 * h);
        const uint32_t row = divu32(sp, div_spr), seg = sp - row * spr;
        // scale byte of block 32 seg + 8 h + lane / 4: word 8 seg + 2 h + lane / 16 of the row
        uint8_t *sfp = sf + sf_word_offset(row, (int64_t)seg * 8 + (lane >> 4), KB) + ((lane >> 2) & 3);
        uint2 *dst = reinterpret_cast<uint2 *>(codes + e0) + lane;
        const uint64_t chunk0 = ((uint64_t)sp << 7) + lane;
#pragma unroll
        for (int h = 0; h < 4; h++) {
            const uint32_t w[4] = {raw[h].x, raw[h].y, raw[h].z, raw[h].w};
            uint32_t sb;
            if (SR) {
                uint32_t a[4];
                uint32_t m = bf16_chunk_absmax(w, a);
                m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
                m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
                sb = mx_scale_code_bf16(m);
                const uint2 q = mx_sr8_bf16(w, a, sb, mx_draws(chunk0 + 32 * h, keys, stream_id));
                dst[32 * h] = (m == 0u) ? make_uint2(0u, 0u) : q;
            } else {
                float v[8];
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    v[2 * i] = bf16_lo(w[i]);
                    v[2 * i + 1] = bf16_hi(w[i]);
                }
                float m = fmax3(fmax3(fabsf(v[0]), fabsf(v[1]), fabsf(v[2])),
                                fmax3(fabsf(v[3]), fabsf(v[4]), fabsf(v[5])), fmaxf(fabsf(v[6]), fabsf(v[7])));
                m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
                m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
                sb = mx_scale_code(m);
                dst[32 * h] = mx_encode8<false>(v, m == 0.0f, sb, 0, keys, 0u);
            }
            if (sf_lane) sfp[h * 1024] = (uint8_t)sb;
        }
    }
}

// Column-wise (output [K, M] = quantization of the transpose, blocks of 32
// along M) from bf16.  A warp covers 32 input rows x 64 input columns with
// no shared memory: lane l = 4 kg + mg loads the 8 x 8 piece of rows
// 8 mg .. 8 mg + 7 and columns 8 kg .. 8 kg + 7 (each warp-wide load reads
// 128 contiguous bytes of four rows), which holds, per column, one output
// chunk of 8 consecutive m; the four lanes with the same kg share that
// column's block of 32 (two-step shuffle max).  Warp tiles run m-fastest, so
// consecutive warps write adjacent 32-byte pieces of each output row.
// I: the output index type (uint32_t when M * K < 2^31: the code offset,
// the Philox counter and the scale offset in single 32-bit instructions).
template <bool SR, typename I>
__global__ void __launch_bounds__(256) quant_mxfp8_col_kernel(
    const uint16_t *__restrict__ xin, int64_t M, int64_t K, int64_t ldx, uint32_t ntile, DivU32 div_mt,
    const __grid_constant__ PhiloxKeys keys, uint32_t stream_id, uint8_t *__restrict__ codes,
    uint8_t *__restrict__ sf) {
    const int lane = threadIdx.x & 31, kg = lane >> 2, mg = lane & 3;
    const uint32_t mt_n = (uint32_t)(M >> 5);
    const int64_t MB = M >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    for (uint32_t t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < ntile; t += nwarps) {
        const uint32_t kt = divu32(t, div_mt), mt = t - kt * mt_n;
        const int64_t m0 = (int64_t)mt * 32 + mg * 8, k0 = (int64_t)kt * 64 + kg * 8;
        const bool kvalid = k0 < K;  // K % 8 == 0: a lane's 8 columns are all in or all out
        // w[i][p]: columns 2p, 2p + 1 of row m0 + i (low half: the even column)
        uint32_t w[8][4];
        const uint16_t *x = xin + m0 * ldx + k0;
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const uint4 r = kvalid ? __ldg(reinterpret_cast<const uint4 *>(x + i * ldx)) : make_uint4(0, 0, 0, 0);
            w[i][0] = r.x; w[i][1] = r.y; w[i][2] = r.z; w[i][3] = r.w;
        }
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const I k = (I)k0 + (I)j;
            const I o = k * (I)M + (I)m0;  // output offset of this chunk
            uint2 q;
            uint32_t sb;
            bool zero;
            if (SR) {
                // rows 2i, 2i + 1 of column j as one bf16 pair
                uint32_t p[4], a[4];
#pragma unroll
                for (int i = 0; i < 4; i++)
                    p[i] = __byte_perm(w[2 * i][j >> 1], w[2 * i + 1][j >> 1], (j & 1) ? 0x7632u : 0x5410u);
                uint32_t m = bf16_chunk_absmax(p, a);
                m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
                m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
                sb = mx_scale_code_bf16(m);
                q = mx_sr8_bf16(p, a, sb, mx_draws((uint64_t)(o >> 3), keys, stream_id));
                zero = m == 0u;
            } else {
                float v[8];
#pragma unroll
                for (int i = 0; i < 8; i++) v[i] = (j & 1) ? bf16_hi(w[i][j >> 1]) : bf16_lo(w[i][j >> 1]);
                float m = fmax3(fmax3(fabsf(v[0]), fabsf(v[1]), fabsf(v[2])),
                                fmax3(fabsf(v[3]), fabsf(v[4]), fabsf(v[5])), fmaxf(fabsf(v[6]), fabsf(v[7])));
                m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
                m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
                sb = mx_scale_code(m);
                q = mx_encode8<false>(v, false, sb, 0, keys, 0u);
                zero = m == 0.0f;
            }
            if (zero) q = make_uint2(0u, 0u);
            if (kvalid) {
                *reinterpret_cast<uint2 *>(codes + (size_t)o) = q;
                if (mg == 0) {
                    // sf_offset(k, m0 / 32, MB) in the index type
                    const I b = (I)(m0 >> 5), bt = ((I)MB + 3) >> 2;
                    const I so = (((k >> 7) * bt + (b >> 2)) << 9) + ((k & 31) << 4) + (((k >> 5) & 3) << 2) + (b & 3);
                    sf[(size_t)so] = (uint8_t)sb;
                }
            }
        }
    }
}

// Dequantize -> transpose -> requantize of a row-wise MXFP8 tensor.  The
// column kernel's warp tile: lane l = 4 kg + mg holds rows 8 mg .. 8 mg + 7
// and columns 8 kg .. 8 kg + 7 (one 8-byte code load and one E8M0 byte per
// row: the 8 columns sit in one input block).  Each value is decoded exactly
// (E4M3 -> f16 -> fp32, times its power-of-two row scale) and requantized
// with the column block's scale; a chunk whose rescaled values are all E4M3
// values (the common case: an E4M3 value times a power of two) needs no
// rounding and takes the nearest-even conversion without drawing.
// I: the index type of offsets and Philox counters (uint32_t when the
// tensor has fewer than 2^31 elements: single 32-bit instructions).
template <bool SR, typename I>
__global__ void __launch_bounds__(256) requant_transpose_kernel(
    const uint8_t *__restrict__ codes_in, const uint8_t *__restrict__ sf_in, int64_t M, int64_t K, uint32_t ntile,
    DivU32 div_mt, const __grid_constant__ PhiloxKeys keys, uint32_t stream_id, uint8_t *__restrict__ codes,
    uint8_t *__restrict__ sf) {
    const int lane = threadIdx.x & 31, kg = lane >> 2, mg = lane & 3;
    const uint32_t mt_n = (uint32_t)(M >> 5);
    const int64_t MB = M >> 5, KB = K >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    for (uint32_t t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < ntile; t += nwarps) {
        const uint32_t kt = divu32(t, div_mt), mt = t - kt * mt_n;
        const int64_t m0 = (int64_t)mt * 32 + mg * 8, k0 = (int64_t)kt * 64 + kg * 8;
        const bool kvalid = k0 < K;  // K % 32 == 0: a lane's 8 columns are all in or all out
        uint32_t w[8][2];
        float sc[8];
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const uint2 r = kvalid ? __ldg(reinterpret_cast<const uint2 *>(codes_in + (size_t)((I)(m0 + i) * (I)K + (I)k0))) : make_uint2(0, 0);
            w[i][0] = r.x;
            w[i][1] = r.y;
            sc[i] = kvalid ? exp2i((int)__ldg(sf_in + (size_t)sf_offset_t<I>((I)(m0 + i), (I)(k0 >> 5), (I)KB)) - 127) : 0.0f;
        }
        float odd[8];  // column j + 1, decoded with column j
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const I k = (I)k0 + (I)j;
            const I o = k * (I)M + (I)m0;  // output offset of this chunk
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; i++) {
                if ((j & 1) == 0) {
                    float e0, e1;
                    e4m3x2_to_f32(w[i][j >> 2] >> (8 * (j & 3)), e0, e1);
                    v[i] = __fmul_rn(e0, sc[i]);
                    odd[i] = __fmul_rn(e1, sc[i]);
                } else {
                    v[i] = odd[i];
                }
            }
            float m = fmax3(fmax3(fabsf(v[0]), fabsf(v[1]), fabsf(v[2])), fmax3(fabsf(v[3]), fabsf(v[4]), fabsf(v[5])),
                            fmaxf(fabsf(v[6]), fabsf(v[7])));
            m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
            m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
            const uint32_t sb = mx_scale_code(m);
            const uint2 q = mx_encode8<SR, true>(v, m == 0.0f, sb, (uint64_t)(o >> 3), keys, stream_id);
            if (kvalid) {
                *reinterpret_cast<uint2 *>(codes + (size_t)o) = q;
                if (mg == 0) sf[(size_t)sf_offset_t<I>(k, (I)(m0 >> 5), (I)MB)] = (uint8_t)sb;
            }
        }
    }
}

// Row-wise and column-wise MXFP8 of one bf16 tensor in one pass (the
// backward pass needs dY both ways): the column kernel's warp tile (32 rows
// x 64 columns, lane l = 4 kg + mg holding rows 8 mg .. 8 mg + 7 and columns
// 8 kg .. 8 kg + 7) also yields, per held row, one row-wise chunk of 8; the
// four lanes mg, mg + 4, mg + 8, mg + 12 (and likewise the upper four kg)
// hold one row block of 32, reduced with shuffles over lane bits 2 and 3.
// Row output: codes_r [M][K], SR draws of row * K + col with stream_r;
// column output: codes_c [K][M], draws of k * M + m with stream_c.
// I: the index type of offsets and Philox counters (uint32_t when the
// tensor has fewer than 2^31 elements: single 32-bit instructions).
template <bool SR, typename I>
__global__ void __launch_bounds__(256) quant_mxfp8_rowcol_kernel(
    const uint16_t *__restrict__ x, int64_t M, int64_t K, int64_t ldx, uint32_t ntile, DivU32 div_mt,
    const __grid_constant__ PhiloxKeys keys, uint32_t stream_r, uint32_t stream_c, uint8_t *__restrict__ codes_r,
    uint8_t *__restrict__ sf_r, uint8_t *__restrict__ codes_c, uint8_t *__restrict__ sf_c) {
    const int lane = threadIdx.x & 31, kg = lane >> 2, mg = lane & 3;
    const uint32_t mt_n = (uint32_t)(M >> 5);
    const int64_t MB = M >> 5, KB = K >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    for (uint32_t t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < ntile; t += nwarps) {
        const uint32_t kt = divu32(t, div_mt), mt = t - kt * mt_n;
        const int64_t m0 = (int64_t)mt * 32 + mg * 8, k0 = (int64_t)kt * 64 + kg * 8;
        const bool kvalid = k0 < K;  // K % 32 == 0: a row block of four lanes is all in or all out
        uint32_t w[8][4];
        const uint16_t *xp = x + m0 * ldx + k0;
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const uint4 r = kvalid ? __ldg(reinterpret_cast<const uint4 *>(xp + i * ldx)) : make_uint4(0, 0, 0, 0);
            w[i][0] = r.x; w[i][1] = r.y; w[i][2] = r.z; w[i][3] = r.w;
        }
        // ---- row-wise: row m0 + i, columns k0 .. k0 + 7
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const I row = (I)m0 + (I)i;
            const I orow = row * (I)K + (I)k0;  // row-wise output offset
            uint32_t sb;
            uint2 q;
            if (SR) {
                uint32_t a[4];
                uint32_t m = bf16_chunk_absmax(w[i], a);
                m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
                m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 8));
                sb = mx_scale_code_bf16(m);
                q = mx_sr8_bf16(w[i], a, sb, mx_draws((uint64_t)(orow >> 3), keys, stream_r));
                if (m == 0u) q = make_uint2(0u, 0u);
            } else {
                float v[8];
#pragma unroll
                for (int p = 0; p < 4; p++) {
                    v[2 * p] = bf16_lo(w[i][p]);
                    v[2 * p + 1] = bf16_hi(w[i][p]);
                }
                float m = fmax3(fmax3(fabsf(v[0]), fabsf(v[1]), fabsf(v[2])),
                                fmax3(fabsf(v[3]), fabsf(v[4]), fabsf(v[5])), fmaxf(fabsf(v[6]), fabsf(v[7])));
                m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
                m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 8));
                sb = mx_scale_code(m);
                q = mx_encode8<false>(v, m == 0.0f, sb, 0, keys, 0u);
            }
            if (kvalid) {
                *reinterpret_cast<uint2 *>(codes_r + (size_t)orow) = q;
                if ((kg & 3) == 0) sf_r[(size_t)sf_offset_t<I>(row, (I)(k0 >> 5), (I)KB)] = (uint8_t)sb;
            }
        }
        // ---- column-wise: column k0 + j, rows m0 .. m0 + 7
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const I k = (I)k0 + (I)j;
            const I o = k * (I)M + (I)m0;  // column-wise output offset
            uint32_t sb;
            uint2 q;
            if (SR) {
                uint32_t p[4], a[4];
#pragma unroll
                for (int i = 0; i < 4; i++)
                    p[i] = __byte_perm(w[2 * i][j >> 1], w[2 * i + 1][j >> 1], (j & 1) ? 0x7632u : 0x5410u);
                uint32_t m = bf16_chunk_absmax(p, a);
                m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
                m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
                sb = mx_scale_code_bf16(m);
                q = mx_sr8_bf16(p, a, sb, mx_draws((uint64_t)(o >> 3), keys, stream_c));
                if (m == 0u) q = make_uint2(0u, 0u);
            } else {
                float v[8];
#pragma unroll
                for (int i = 0; i < 8; i++) v[i] = (j & 1) ? bf16_hi(w[i][j >> 1]) : bf16_lo(w[i][j >> 1]);
                float m = fmax3(fmax3(fabsf(v[0]), fabsf(v[1]), fabsf(v[2])),
                                fmax3(fabsf(v[3]), fabsf(v[4]), fabsf(v[5])), fmaxf(fabsf(v[6]), fabsf(v[7])));
                m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
                m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
                sb = mx_scale_code(m);
                q = mx_encode8<false>(v, m == 0.0f, sb, 0, keys, 0u);
            }
            if (kvalid) {
                *reinterpret_cast<uint2 *>(codes_c + (size_t)o) = q;
                if (mg == 0) sf_c[(size_t)sf_offset_t<I>(k, (I)(m0 >> 5), (I)MB)] = (uint8_t)sb;
            }
        }
    }
}

// NVFP4 -> MXFP8 column-wise: the NVFP4 tensor [R][C] (codes [R][C/2],
// swizzled E4M3 scales for R rows x C/16 blocks, s_g on the device) is
// decoded to binary32 as RN(RN(E2M1 * s_b) * s_g) (the first product is
// exact), transposed and quantized to MXFP8 with blocks of 32 along R.  The
// column kernel's warp tile: lane l = 4 kg + mg holds rows 8 mg .. 8 mg + 7
// and columns 8 kg .. 8 kg + 7 (one 32-bit code load and one scale byte per
// row: the 8 columns sit in one 16-block); the four lanes of a kg share the
// output block of column 8 kg + j.
// I: the index type of offsets and Philox counters (uint32_t when the
// tensor has fewer than 2^31 elements: single 32-bit instructions).
template <bool SR, typename I>
__global__ void __launch_bounds__(256) requant_nvfp4_mxfp8_kernel(
    const uint8_t *__restrict__ codes_in, const uint8_t *__restrict__ sf_in, const float *gs, int64_t R, int64_t C,
    uint32_t ntile, DivU32 div_mt, const __grid_constant__ PhiloxKeys keys, uint32_t stream_id,
    uint8_t *__restrict__ codes, uint8_t *__restrict__ sf) {
    const int lane = threadIdx.x & 31, kg = lane >> 2, mg = lane & 3;
    const uint32_t mt_n = (uint32_t)(R >> 5);
    const int64_t RB = R >> 5, CB16 = C >> 4;
    const float s_g = *gs;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    for (uint32_t t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < ntile; t += nwarps) {
        const uint32_t kt = divu32(t, div_mt), mt = t - kt * mt_n;
        const int64_t m0 = (int64_t)mt * 32 + mg * 8, k0 = (int64_t)kt * 64 + kg * 8;
        const bool kvalid = k0 < C;  // C % 16 == 0: a lane's 8 columns are all in or all out
        uint32_t w[8];               // w[i]: the 8 codes of row m0 + i
        float sbv[8];                // its block scale
#pragma unroll
        for (int i = 0; i < 8; i++) {
            w[i] = kvalid ? __ldg(reinterpret_cast<const uint32_t *>(codes_in + (size_t)((I)(m0 + i) * (I)(C >> 1) + (I)(k0 >> 1)))) : 0u;
            sbv[i] = kvalid ? e4m3_to_f32(__ldg(sf_in + (size_t)sf_offset_t<I>((I)(m0 + i), (I)(k0 >> 4), (I)CB16))) : 0.0f;
        }
        auto column = [&](int j, const float (&c)[8]) {
            const I k = (I)k0 + (I)j;
            const I o = k * (I)R + (I)m0;  // output offset of this chunk
            float m = fmax3(fmax3(fabsf(c[0]), fabsf(c[1]), fabsf(c[2])), fmax3(fabsf(c[3]), fabsf(c[4]), fabsf(c[5])),
                            fmaxf(fabsf(c[6]), fabsf(c[7])));
            m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
            m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
            const uint32_t sb = mx_scale_code(m);
            const uint2 q = mx_encode8<SR, false, true>(c, m == 0.0f, sb, (uint64_t)(o >> 3), keys, stream_id);
            if (kvalid) {
                *reinterpret_cast<uint2 *>(codes + (size_t)o) = q;
                if (mg == 0) sf[(size_t)sf_offset_t<I>(k, (I)(m0 >> 5), (I)RB)] = (uint8_t)sb;
            }
        };
        // columns 2 jj and 2 jj + 1 (byte jj of every row), decoded as needed
#pragma unroll
        for (int jj = 0; jj < 4; jj++) {
            float ce[8], co[8];
#pragma unroll
            for (int i = 0; i < 8; i++) {
                float lo, hi;
                e2m1x2_to_f32(w[i] >> (8 * jj), lo, hi);
                ce[i] = __fmul_rn(__fmul_rn(lo, sbv[i]), s_g);
                co[i] = __fmul_rn(__fmul_rn(hi, sbv[i]), s_g);
            }
            column(2 * jj, ce);
            column(2 * jj + 1, co);
        }
    }
}

// ===================================================================== MXFP4
// E2M1 elements in blocks of 32 along K with one E8M0 scale 2^E,
// E = clamp(floor(log2 amax) - 2, -127, 127) (2 is the exponent of E2M1's
// largest value, 6 = 1.5 * 2^2): code max(exponent field - 2, 0), the same
// branch-free form as the MXFP8 code with 2 in place of 8.
BSQ_DEV uint32_t mx4_scale_code(float m) {
    const int f = (int)(__float_as_uint(m) >> 23);
    return (uint32_t)max(f - 2, 0);
}

// Stochastic rounding of s to an E2M1 code (sign bit 3) with the 16-bit draw
// r16: round the magnitude a = min(|s|, 6) up to the next E2M1 value iff
// r16 * 2^-16 < frac.  For a >= 1 the E2M1 neighbour below a is a with its
// low 22 bits cleared (one mantissa bit) and frac = low22 / 2^22, so the test
// is the integer 64 r16 < low22 and rounding up adds 1 << 22; the code is then
// (bits >> 22) - 252 (exponent - 127 + 1, and the mantissa bit).  Below 1 the
// spacing is 0.5: t = 2a, frac = t - floor(t) (both exact), code floor(t) +
// up (0, 0.5 or 1.0).
BSQ_DEV uint32_t e2m1_sr(float s, uint32_t r16) {
    const uint32_t sgn = (__float_as_uint(s) >> 28) & 8u;
    const float a = fminf(fabsf(s), 6.0f);
    uint32_t mag;
    if (a >= 1.0f) {
        const uint32_t b = __float_as_uint(a);
        const uint32_t up = ((r16 << 6) < (b & 0x3FFFFFu)) ? 0x400000u : 0u;
        mag = (((b & ~0x3FFFFFu) + up) >> 22) - 252u;
    } else {
        const float t = __fmul_rn(a, 2.0f);
        const float f = floorf(t);
        const float frac = __fsub_rn(t, f);
        mag = (uint32_t)f + ((__fmul_rn((float)r16, 1.0f / 65536.0f) < frac) ? 1u : 0u);
    }
    return sgn | mag;
}

// The 8 nibbles of one chunk (element 2j in the low nibble of byte j): s =
// v * 2^-E (exact), then nearest-even with saturation at +-6 (the satfinite
// conversion gives +-6 past 6, the same as clamping first) or stochastic
// rounding with the draws of one Philox call (element i: half i & 1 of word
// i / 2).  A zero block stores +0 codes.
template <bool SR>
BSQ_DEV uint32_t mx4_encode8(const float v[8], bool zero, uint32_t sb, uint64_t chunk, const PhiloxKeys &keys,
                             uint32_t stream_id) {
    float s[8];
    mx_scale8(v, __uint_as_float((254u - sb) << 23), s);
    uint32_t q;
    if (SR) {
        const uint4 r = mx_draws(chunk, keys, stream_id);
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
        q = 0u;
#pragma unroll
        for (int i = 0; i < 8; i++) q |= e2m1_sr(s[i], (i & 1) ? (w[i >> 1] >> 16) : (w[i >> 1] & 0xFFFFu)) << (4 * i);
    } else {
        q = cvt_e2m1x8(s);
    }
    return zero ? 0u : q;
}

// Row-wise MXFP4: one thread per 8 elements, 4 lanes per block of 32 (two
// shuffles for the block maximum), rows mapped to lanes as in the MXFP8 row
// kernel; one 32-bit code store per chunk, the scale bytes of 4 blocks
// packed into one 32-bit store when a row holds a multiple of 4 blocks.
// I: the index type of the per-chunk offsets and Philox counters (uint32_t
// when M * ldx < 2^31: single 32-bit instructions).
template <bool SR, typename I>
__global__ void __launch_bounds__(256) quant_mxfp4_row_kernel(
    const uint16_t *__restrict__ x, int64_t M, int64_t K, int64_t ldx, const __grid_constant__ PhiloxKeys keys,
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
            load8_bf16(x + (size_t)((I)rr * (I)ldx + (I)cc * 8), v);
            float m = fmax3(fmax3(fabsf(v[0]), fabsf(v[1]), fabsf(v[2])), fmax3(fabsf(v[3]), fabsf(v[4]), fabsf(v[5])),
                            fmaxf(fabsf(v[6]), fabsf(v[7])));
            m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
            m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
            const uint32_t sb = mx4_scale_code(m);
            const I o = (I)rr * (I)K + (I)cc * 8;  // element offset of this chunk
            const uint32_t q = mx4_encode8<SR>(v, m == 0.0f, sb, (uint64_t)(o >> 3), keys, stream_id);
            if (valid) *reinterpret_cast<uint32_t *>(codes + (size_t)(o >> 1)) = q;
            const int64_t kb = cc >> 2;
            if (pack4) {
                const uint32_t b1 = __shfl_down_sync(0xFFFFFFFFu, sb, 4);
                const uint32_t b2 = __shfl_down_sync(0xFFFFFFFFu, sb, 8);
                const uint32_t b3 = __shfl_down_sync(0xFFFFFFFFu, sb, 12);
                if (valid && (lane & 15) == 0)
                    *reinterpret_cast<uint32_t *>(sf + (size_t)sf_word_offset_t<I>((I)rr, (I)(kb >> 2), (I)KB)) =
                        sb | (b1 << 8) | (b2 << 16) | (b3 << 24);
            } else if (valid && (lane & 3) == 0) {
                sf[(size_t)sf_offset_t<I>((I)rr, (I)kb, (I)KB)] = (uint8_t)sb;
            }
        }
    }
}

// Row-wise MXFP4 for a contiguous tensor whose rows hold a multiple of 1024
// elements: the MXFP8 span kernel's mapping (a warp per 1024-element span of
// one row, lane l loads the 8-element chunks l, l + 32, l + 64, l + 96, four
// 16-byte loads in flight; lanes 4j .. 4j + 3 share a block of 32), with one
// 32-bit code store per chunk.  The SR draw index of a chunk is its flat
// position, as in quant_mxfp4_row_kernel.
template <bool SR>
__global__ void __launch_bounds__(256) quant_mxfp4_row_span_kernel(
    const uint16_t *__restrict__ x, uint32_t nspan, int64_t K, DivU32 div_spr, const __grid_constant__ PhiloxKeys keys,
    uint32_t stream_id, uint8_t *__restrict__ codes, uint8_t *__restrict__ sf) {
    const int lane = threadIdx.x & 31;
    const uint32_t spr = (uint32_t)(K >> 10);  // spans per row
    const int64_t KB = K >> 5;
    const uint32_t nwarps = (gridDim.x * blockDim.x) >> 5;
    const bool sf_lane = (lane & 3) == 0;
    for (uint32_t sp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; sp < nspan; sp += nwarps) {
        const int64_t e0 = (int64_t)sp << 10;
        const uint4 *src = reinterpret_cast<const uint4 *>(x + e0) + lane;
        uint4 raw[4];
#pragma unroll
        for (int h = 0; h < 4; h++) raw[h] = __ldg(src + 32 * h);
        const uint32_t row = divu32(sp, div_spr), seg = sp - row * spr;
        // scale byte of block 32 seg + 8 h + lane / 4: word 8 seg + 2 h + lane / 16 of the row
        uint8_t *sfp = sf + sf_word_offset(row, (int64_t)seg * 8 + (lane >> 4), KB) + ((lane >> 2) & 3);
        uint32_t *dst = reinterpret_cast<uint32_t *>(codes + (e0 >> 1)) + lane;
        const uint64_t chunk0 = ((uint64_t)sp << 7) + lane;
#pragma unroll
        for (int h = 0; h < 4; h++) {
            const uint32_t w[4] = {raw[h].x, raw[h].y, raw[h].z, raw[h].w};
            float v[8];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                v[2 * i] = bf16_lo(w[i]);
                v[2 * i + 1] = bf16_hi(w[i]);
            }
            float m = fmax3(fmax3(fabsf(v[0]), fabsf(v[1]), fabsf(v[2])), fmax3(fabsf(v[3]), fabsf(v[4]), fabsf(v[5])),
                            fmaxf(fabsf(v[6]), fabsf(v[7])));
            m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
            m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
            const uint32_t sb = mx4_scale_code(m);
            dst[32 * h] = mx4_encode8<SR>(v, m == 0.0f, sb, chunk0 + 32 * h, keys, stream_id);
            if (sf_lane) sfp[h * 1024] = (uint8_t)sb;
        }
    }
}

// ===================================================================== NVFP4, stochastic rounding
// NVFP4 with the elements rounded stochastically: block scales and s_g as
// in the nearest-even kernels above; each element q = y * r (y = RN(u / 4)
// with the RHT, then RN(y * r): the definition's order also where y is
// subnormal, since a tiny q can still round up to 0.5), clamped to +-6 and
// rounded by e2m1_sr with the draws of output elements idx0 .. idx0 + 15
// (two Philox calls; idx0 = row * K + 16 * block).
template <bool RHT>
BSQ_DEV uint2 nv_codes_sr(const f32x2 P[8], float r, uint64_t idx0, const PhiloxKeys &keys, uint32_t stream_id) {
    f32x2 Q[8];
#pragma unroll
    for (int k = 0; k < 8; k++) Q[k] = P[k];
    if (RHT) pairs_scale(Q, 0.25f);
    const f32x2 R = f2_pack(r, r);
    float q[16];
#pragma unroll
    for (int k = 0; k < 8; k++) f2_unpack(f2_mul(Q[k], R), q[2 * k], q[2 * k + 1]);
    uint32_t out[2];
#pragma unroll
    for (int h = 0; h < 2; h++) {
        const uint4 rw = mx_draws((idx0 >> 3) + h, keys, stream_id);
        const uint32_t w[4] = {rw.x, rw.y, rw.z, rw.w};
        uint32_t word = 0u;
#pragma unroll
        for (int i = 0; i < 8; i++)
            word |= e2m1_sr(q[8 * h + i], (i & 1) ? (w[i >> 1] >> 16) : (w[i >> 1] & 0xFFFFu)) << (4 * i);
        out[h] = word;
    }
    return make_uint2(out[0], out[1]);
}

// 1x16 blocks, rows (optionally gathered): one thread per block, rows mapped
// to lanes as in quant_nvfp4_1d_kernel.
// I: the index type of the per-block offsets and Philox counters (uint32_t
// when the output holds fewer than 2^31 elements).
template <bool RHT, bool GATHER, typename I>
__global__ void __launch_bounds__(256) quant_nvfp4_sr_1d_kernel(
    const uint16_t *__restrict__ x, int64_t M, int64_t K, int64_t ldx, uint32_t mask,
    const int32_t *__restrict__ row_index, const float *scale_src, int src_is_amax, float *gs_out, int write_gs,
    const __grid_constant__ PhiloxKeys keys, uint32_t stream_id, uint8_t *__restrict__ codes,
    uint8_t *__restrict__ sf, RowMap map) {
    __shared__ float den_tab[128], rcp_tab[128];
    const int64_t KB = K >> 4;
    const bool pack4 = (KB & 3) == 0;
    const float s_g = src_is_amax ? global_scale_of(*scale_src) : *scale_src;
    if (write_gs && blockIdx.x == 0 && threadIdx.x == 0) *gs_out = s_g;
    const NvScale c = nv_scale_setup(s_g, den_tab, rcp_tab);
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
        for (int64_t kb0 = 0; kb0 < KB; kb0 += lpr) {
            const int64_t kb = kb0 + lk;
            const bool valid = row_ok && kb < KB;
            const int64_t kk = kb < KB ? kb : KB - 1;
            uint32_t w[8];
            load_words16(rp + (size_t)((I)kk * 16), w);
            f32x2 P[8];
            if (RHT) rht16_u_words(w, sw, P);
            else words_to_pairs(w, P);
            const float mu = pairs_absmax3(P);
            const uint32_t sb = nv_scale_code(RHT ? __fmul_rn(mu, 0.25f) : mu, 6.0f, c.c6, c);
            const uint2 cd = sb ? nv_codes_sr<RHT>(P, rcp_tab[sb], (uint64_t)((I)rr * (I)K + (I)kk * 16), keys, stream_id)
                                : make_uint2(0u, 0u);
            if (valid) *reinterpret_cast<uint2 *>(codes + (size_t)((I)rr * (I)(K >> 1) + (I)kb * 8)) = cd;
            store_sf_t<I>(sf, valid, sb, (I)rr, (I)kb, (I)KB, pack4);
        }
    }
}

// 16x16 tiles: the tile mapping of quant_nvfp4_2d_kernel (a warp covers one
// 16-row tile row and eight blocks; lane l: row l % 16, blocks 4 (l / 16) ..
// 4 (l / 16) + 3; tile amax over a half-warp).
template <bool RHT>
__global__ void __launch_bounds__(256) quant_nvfp4_sr_2d_kernel(
    const uint16_t *__restrict__ x, int64_t M, int64_t K, int64_t ldx, uint32_t mask, const float *scale_src,
    int src_is_amax, float *gs_out, int write_gs, const __grid_constant__ PhiloxKeys keys, uint32_t stream_id,
    uint8_t *__restrict__ codes, uint8_t *__restrict__ sf) {
    __shared__ float den_tab[128], rcp_tab[128];
    const float s_g = src_is_amax ? global_scale_of(*scale_src) : *scale_src;
    if (write_gs && blockIdx.x == 0 && threadIdx.x == 0) *gs_out = s_g;
    const NvScale c = nv_scale_setup(s_g, den_tab, rcp_tab);
    uint32_t sw[8];
    rht_sign_words(mask, sw);
    const int64_t KB = K >> 4;
    const int64_t k8 = (KB + 7) >> 3;
    const int64_t tasks = (M >> 4) * k8;
    const int lane = threadIdx.x & 31;
    const int r16 = lane & 15, hw = lane >> 4;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t task = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); task < tasks; task += warps) {
        const int64_t rt = task / k8, g8 = task - rt * k8;
        const int64_t row = rt * 16 + r16;
        const int64_t kb0 = g8 * 8 + 4 * hw;
        const uint16_t *rp = x + row * ldx;
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const int64_t kb = kb0 + i;
            const bool v = kb < KB;  // uniform over the half-warp
            uint32_t w[8];
            load_words16(rp + (v ? kb : 0) * 16, w);
            f32x2 P[8];
            if (RHT) rht16_u_words(w, sw, P);
            else words_to_pairs(w, P);
            float mu = v ? pairs_absmax3(P) : 0.0f;
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) mu = fmaxf(mu, __shfl_xor_sync(0xFFFFFFFFu, mu, o));
            const uint32_t sb = nv_scale_code(RHT ? __fmul_rn(mu, 0.25f) : mu, 6.0f, c.c6, c);
            const uint2 cd = (sb && v) ? nv_codes_sr<RHT>(P, rcp_tab[sb], (uint64_t)(row * K + kb * 16), keys,
                                                          stream_id)
                                       : make_uint2(0u, 0u);
            if (v) {
                *reinterpret_cast<uint2 *>(codes + row * (K >> 1) + kb * 8) = cd;
                sf[sf_offset(row, kb, KB)] = (uint8_t)sb;
            }
        }
    }
}

// ===================================================================== S2F6 (MoE combine)
// Block-scaled S2F6 for the combine exchange: two's-complement fixed point
// with six fraction bits (q / 64, q in [-128, 127]), one E8M0 scale 2^E per
// 32 values with E = floor(log2 block_amax) (so block_amax / 2^E is in
// [1, 2)), after the 16-point RHT.  One thread per group of 16 (the RHT
// group), two lanes per block of 32; codes [M][K] int8 and scales [M][K/32]
// row-major (a transport format, not an MMA layout).

// y * 2^k for a power-of-two scaling that stays exact (or rounds once into
// the subnormal range), for k in [-149, 254].
BSQ_DEV float mul_pow2(float y, int k) {
    if (k > 127) return __fmul_rn(__fmul_rn(y, 0x1p64f), exp2i(k - 64));
    return __fmul_rn(y, exp2i(k));
}

template <bool RHT>
__global__ void __launch_bounds__(256) quant_s2f6_kernel(const uint16_t *__restrict__ x, int64_t M, int64_t K,
                                                         int64_t ldx, uint32_t mask, int8_t *__restrict__ codes,
                                                         uint8_t *__restrict__ sf, RowMap map) {
    const int64_t KG = K >> 4;
    uint32_t sw[8];
    rht_sign_words(mask, sw);
    const int lpr = 1 << map.lpr_shift;
    const int rpi = 256 >> map.lpr_shift;
    const int sub = threadIdx.x >> map.lpr_shift, lk = threadIdx.x & (lpr - 1);
    for (int64_t r0 = (int64_t)blockIdx.x * rpi; r0 < M; r0 += (int64_t)gridDim.x * rpi) {
        const int64_t row = r0 + sub;
        const bool row_ok = row < M;
        const int64_t rr = row_ok ? row : M - 1;
        for (int64_t g0 = 0; g0 < KG; g0 += lpr) {
            const int64_t g = g0 + lk;
            const bool valid = row_ok && g < KG;   // KG is even: the two lanes of a block agree
            uint32_t w[8];
            load_words16(x + rr * ldx + (g < KG ? g : KG - 1) * 16, w);
            f32x2 P[8];
            if (RHT) {
                rht16_u_words(w, sw, P);
                pairs_scale(P, 0.25f);
            } else {
                words_to_pairs(w, P);
            }
            float m = pairs_absmax3(P);
            m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
            const int E = m == 0.0f ? 0 : min(max(floor_log2(m), -127), 127);
            float v[16];
#pragma unroll
            for (int k = 0; k < 8; k++) f2_unpack(P[k], v[2 * k], v[2 * k + 1]);
            uint32_t q[4];
#pragma unroll
            for (int k = 0; k < 4; k++) {
                uint32_t word = 0u;
#pragma unroll
                for (int b = 0; b < 4; b++) {
                    const int iq = min(max(__float2int_rn(mul_pow2(v[4 * k + b], 6 - E)), -128), 127);
                    word |= ((uint32_t)iq & 0xFFu) << (8 * b);
                }
                q[k] = m == 0.0f ? 0u : word;
            }
            if (valid) {
                *reinterpret_cast<uint4 *>(codes + rr * K + g * 16) = make_uint4(q[0], q[1], q[2], q[3]);
                if ((g & 1) == 0) sf[rr * (K >> 5) + (g >> 1)] = m == 0.0f ? 0 : (uint8_t)(E + 127);
            }
        }
    }
}

// The receiver: token t's output, group g of 16 = inverse RHT of the sum over
// the token's listed rows (in list order) of weight * value, each product and
// addition one RN operation; x = 1/4 * D * H16 * acc (butterflies of stride
// 1, 2, 4, 8, RN), rounded once to bf16.  One thread per (token, group).
__global__ void __launch_bounds__(256) combine_s2f6_kernel(const int8_t *__restrict__ codes,
                                                           const uint8_t *__restrict__ sf, int64_t K,
                                                           const int32_t *__restrict__ off,
                                                           const int32_t *__restrict__ rows,
                                                           const float *__restrict__ weights, int64_t T,
                                                           uint32_t mask, uint16_t *__restrict__ out, int64_t ldo) {
    const int64_t KG = K >> 4;
    const int64_t n = T * KG;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / KG, g = i - t * KG;
        float acc[16];
#pragma unroll
        for (int k = 0; k < 16; k++) acc[k] = 0.0f;
        const int32_t j1 = __ldg(off + t + 1);
        for (int32_t j = __ldg(off + t); j < j1; j++) {
            const int64_t r = __ldg(rows + j);
            const float wgt = __ldg(weights + j);
            const uint4 cw = __ldg(reinterpret_cast<const uint4 *>(codes + r * K + g * 16));
            const float scale = exp2i((int)__ldg(sf + r * (K >> 5) + (g >> 1)) - 133);
            const uint32_t c4[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
            for (int k = 0; k < 16; k++) {
                const float v = __fmul_rn((float)(int8_t)(c4[k >> 2] >> (8 * (k & 3))), scale);
                acc[k] = __fadd_rn(acc[k], __fmul_rn(wgt, v));
            }
        }
#pragma unroll
        for (int h = 1; h < 16; h <<= 1)
#pragma unroll
            for (int base = 0; base < 16; base += 2 * h)
#pragma unroll
                for (int k = base; k < base + h; k++) {
                    const float a = acc[k], b = acc[k + h];
                    acc[k] = __fadd_rn(a, b);
                    acc[k + h] = __fsub_rn(a, b);
                }
        uint32_t o[8];
#pragma unroll
        for (int k = 0; k < 8; k++) {
            float y0 = __fmul_rn(acc[2 * k], 0.25f), y1 = __fmul_rn(acc[2 * k + 1], 0.25f);
            if ((mask >> (2 * k)) & 1u) y0 = -y0;
            if ((mask >> (2 * k + 1)) & 1u) y1 = -y1;
            __nv_bfloat162 hb = __floats2bfloat162_rn(y0, y1);
            o[k] = *reinterpret_cast<uint32_t *>(&hb);
        }
        uint4 *dst = reinterpret_cast<uint4 *>(out + t * ldo + g * 16);
        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

// ===================================================================== exchange layouts
// Byte-moving kernels for the expert-parallel exchange: rows gathered by an
// index (16-byte pieces), and scale factors between the MMA's swizzled
// layout and plain rows of nblk bytes (the transport form).
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4 *__restrict__ src, int64_t row_vec,
                                                          const int32_t *__restrict__ index, int64_t R,
                                                          uint4 *__restrict__ dst) {
    // one warp per destination row; four 16-byte loads in flight per lane
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < R; row += nwarps) {
        const uint4 *s = src + (int64_t)__ldg(index + row) * row_vec;
        uint4 *d = dst + row * row_vec;
        int64_t v = lane;
        for (; v + 96 < row_vec; v += 128) {
            const uint4 a = __ldg(s + v), b = __ldg(s + v + 32), c = __ldg(s + v + 64), e = __ldg(s + v + 96);
            d[v] = a;
            d[v + 32] = b;
            d[v + 64] = c;
            d[v + 96] = e;
        }
        for (; v < row_vec; v += 32) d[v] = __ldg(s + v);
    }
}

// (i = r nblk + b: the row by a precomputed multiply-shift divider, 32-bit
// indices: the entry points accept rows * nblk < 2^31 only)
__global__ void __launch_bounds__(256) sf_to_rows_kernel(const uint8_t *__restrict__ sf, int64_t rows, int64_t nblk,
                                                         DivU32 div_nblk, uint8_t *__restrict__ out) {
    const uint32_t n = (uint32_t)(rows * nblk), nb = (uint32_t)nblk;
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const uint32_t r = divu32(i, div_nblk), b = i - r * nb;
        out[i] = __ldg(sf + sf_offset(r, b, nblk));
    }
}

// Rows of scale bytes into the swizzled layout; with groups, output row r
// of group e goes to SF row r - row_off[e] + sf_row_off[e] (rows outside
// every group are skipped).
__global__ void __launch_bounds__(256) sf_from_rows_kernel(const uint8_t *__restrict__ in, int64_t rows, int64_t nblk,
                                                           DivU32 div_nblk, int G, const int32_t *__restrict__ row_off,
                                                           const int32_t *__restrict__ sf_off,
                                                           uint8_t *__restrict__ sf) {
    const uint32_t n = (uint32_t)(rows * nblk), nb = (uint32_t)nblk;
    for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const uint32_t r = divu32(i, div_nblk), b = i - r * nb;
        const int64_t sr = G > 0 ? grouped_sf_row(r, G, row_off, sf_off) : (int64_t)r;
        if (sr >= 0) sf[sf_offset(sr, b, nblk)] = __ldg(in + i);
    }
}

// ===================================================================== NVFP4 of gathered rows, by source row
// When the rows to quantize are gathered with repeats (MoE routing sends
// every token to k experts), each output row's codes and scales depend only
// on its source row and s_g.  So the source rows are quantized once and the
// results gathered: a per-row maximum of the source (one warp per row), the
// maximum over the gathered rows (-> s_g), the quantization of the source
// rows, then the code rows and scale words moved to the output.

// rowmax[r] = max |x[r][:]| (after the RHT when enabled): one warp per row.
template <bool RHT>
__global__ void __launch_bounds__(256) row_absmax_kernel(const uint16_t *__restrict__ x, int64_t T, int64_t K,
                                                         int64_t ldx, uint32_t mask, float *__restrict__ rowmax) {
    uint32_t sw[8];
    rht_sign_words(mask, sw);
    const int lane = threadIdx.x & 31;
    const int64_t KB = K >> 4;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < T; r += nw) {
        float m = 0.0f;
        for (int64_t kb = lane; kb < KB; kb += 32) {
            uint32_t w[8];
            load_words16(x + r * ldx + kb * 16, w);
            m = fmaxf(m, block_absmax<RHT>(w, sw));
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (lane == 0) rowmax[r] = m;
    }
}

// max over i < M of rowmax[row_index[i]] into *amax_bits; the last CTA
// writes s_g to *gs_out.
__global__ void __launch_bounds__(256) gathered_max_kernel(const float *__restrict__ rowmax,
                                                           const int32_t *__restrict__ row_index, int64_t M,
                                                           unsigned int *amax_bits, unsigned int *counter,
                                                           float *gs_out) {
    float m = 0.0f;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < M; i += (int64_t)gridDim.x * blockDim.x)
        m = fmaxf(m, __ldg(rowmax + __ldg(row_index + i)));
    block_reduce_atomic_max(m, amax_bits, counter, gs_out);
}

// Scale words of gathered rows: output row i (SF row through the groups, as
// the quantizer maps it) takes source row row_index[i]'s words.
__global__ void __launch_bounds__(256) gather_sf_kernel(const uint8_t *__restrict__ sf_src, int64_t nblk,
                                                        DivU32 div_ng, const int32_t *__restrict__ row_index,
                                                        int64_t M, int G, const int32_t *__restrict__ row_off,
                                                        const int32_t *__restrict__ sf_off, uint8_t *__restrict__ sf) {
    // The destination is written in units of four 512-byte atoms (128 rows x
    // four 4-block groups) per 128 threads: thread t writes word t of each of
    // the unit's atoms, which holds tile row (t >> 2) + 32 (t & 3) (the
    // swizzle puts row r's word at 16 (r % 32) + 4 ((r / 32) % 4)), so each
    // atom's stores are one contiguous run, and the thread's four source
    // words (one row, four groups) are loaded together.  With groups,
    // destination row d of group e (sf_off[e] <= d < sf_off[e] + rows of e)
    // holds routed row d - sf_off[e] + row_off[e]; the padding rows of a
    // group's last tile are not written.
    __shared__ int32_t s_off[1025], s_sfo[1025];
    if (G > 0) {
        for (int i = threadIdx.x; i <= G; i += blockDim.x) {
            s_off[i] = __ldg(row_off + i);
            s_sfo[i] = __ldg(sf_off + i);
        }
        __syncthreads();
    }
    const uint32_t nw4 = (uint32_t)(nblk >> 2), ng = (nw4 + 3) >> 2;  // 4-block groups, units per tile
    const int64_t rows = G > 0 ? (int64_t)s_sfo[G] : M;
    const uint32_t units = (uint32_t)((rows + 127) >> 7) * ng;
    const uint32_t t = threadIdx.x & 127;
    const uint32_t rl = (t >> 2) + 32 * (t & 3);
    for (uint32_t u = blockIdx.x * 2 + (threadIdx.x >> 7); u < units; u += gridDim.x * 2) {
        const uint32_t tile = divu32(u, div_ng), b40 = (u - tile * ng) * 4;
        const int64_t dr = (int64_t)tile * 128 + rl;
        int64_t r = dr;
        bool valid = dr < M;
        if (G > 0) {
            valid = dr >= s_sfo[0];
            if (valid) {
                int lo = 0, hi = G;  // s_sfo[lo] <= dr < s_sfo[hi]: the last group starting at or before dr
                while (hi - lo > 1) {
                    const int mid = (lo + hi) >> 1;
                    if (s_sfo[mid] <= dr) lo = mid; else hi = mid;
                }
                const int64_t in_grp = dr - s_sfo[lo];
                valid = in_grp < (int64_t)(s_off[lo + 1] - s_off[lo]);
                r = s_off[lo] + in_grp;
            }
        }
        if (valid) {
            const int64_t src_row = __ldg(row_index + r);
            const uint8_t *src = sf_src + sf_word_offset(src_row, b40, nblk);  // group b40; b40 + i is 512 i further
            uint8_t *dst = sf + (((size_t)tile * nw4 + b40) << 9) + 4 * t;
            const uint32_t n = nw4 - b40 < 4 ? nw4 - b40 : 4;
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; i++)
                if ((uint32_t)i < n) w[i] = __ldg(reinterpret_cast<const uint32_t *>(src + 512 * i));
#pragma unroll
            for (int i = 0; i < 4; i++)
                if ((uint32_t)i < n) *reinterpret_cast<uint32_t *>(dst + 512 * i) = w[i];
        }
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

// CTAs of `kernel` (256 threads, static shared memory only) that fit on the
// device at once: the grid of the persistent streaming kernels is one full
// wave, so no partial last wave leaves SMs idle.  Kept per kernel and device.
PerDeviceMemo<1024> g_occupancy;

static int current_device() {
    int dev = 0;
    return cudaGetDevice(&dev) == cudaSuccess && dev >= 0 ? dev : 0;
}

template <auto Kern>
static int resident_ctas(int num_sms) {
    const int n = g_occupancy.get(
        reinterpret_cast<const void *>(Kern), current_device(),
        [] {
            int v = 0;
            return cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, Kern, 256, 0) == cudaSuccess ? v : 0;
        },
        [](int v) { return v >= 1; });
    return (n < 1 ? 1 : n) * num_sms;
}

void launch_amax(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, bool rht, uint32_t mask,
                 const int32_t *row_index, unsigned int *amax_bits, unsigned int *counter, float *gs_out,
                 int num_sms, cudaStream_t s) {
    if (!row_index && ldx == K) {
        const int64_t nblk = M * (K >> 4);
#define BSQ_AMF(R, I)                                                                              \
    launch_dependent(amax_flat_kernel<R, I>, grid_for(nblk, 4 * 256, resident_ctas<amax_flat_kernel<R, I>>(num_sms)), \
                     256, 0, s, x, nblk, mask, amax_bits, counter, gs_out)
        if (nblk < (int64_t(1) << 31)) {
            if (rht) BSQ_AMF(true, uint32_t); else BSQ_AMF(false, uint32_t);
        } else {
            if (rht) BSQ_AMF(true, int64_t); else BSQ_AMF(false, int64_t);
        }
#undef BSQ_AMF
        return;
    }
    RowMap map{lpr_shift_for(K >> 4)};
    const int grid = grid_for(M, 256 >> map.lpr_shift, num_sms * 8);
#define BSQ_AMAX(R, G) \
    amax_kernel<R, G><<<grid, 256, 0, s>>>(x, M, K, ldx, mask, row_index, amax_bits, counter, gs_out, map)
    if (rht) { if (row_index) BSQ_AMAX(true, true); else BSQ_AMAX(true, false); }
    else { if (row_index) BSQ_AMAX(false, true); else BSQ_AMAX(false, false); }
#undef BSQ_AMAX
}

void launch_finalize_global_scale(float *gs, cudaStream_t s) { finalize_global_scale_kernel<<<1, 1, 0, s>>>(gs); }

void launch_amax_partials(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, bool rht, uint32_t mask,
                          unsigned int *scratch, float *gs_out, cudaStream_t s) {
    const int64_t nblk = M * (K >> 4);
    const int grid = (int)((nblk + kPartialBlocks - 1) / kPartialBlocks);
    if (rht) amax_partials_kernel<true><<<grid, 256, 0, s>>>(x, M, K, ldx, mask, scratch, gs_out);
    else amax_partials_kernel<false><<<grid, 256, 0, s>>>(x, M, K, ldx, mask, scratch, gs_out);
}

void launch_quant_nvfp4(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, bool block_2d, bool fos,
                        bool rht, uint32_t mask, const int32_t *row_index, int G, const int32_t *row_off,
                        const int32_t *sf_off, const float *scale_src, bool src_is_amax, float *gs_out,
                        bool write_gs, uint8_t *codes, uint8_t *sf, int num_sms, cudaStream_t s) {
    const int sa = src_is_amax ? 1 : 0, wg = write_gs ? 1 : 0;
    if (block_2d) {
        const int64_t tasks = (M >> 4) * (((K >> 4) + 7) >> 3);
        if (rht) {
            const int grid = grid_for(tasks, 8, resident_ctas<quant_nvfp4_2d_kernel<true>>(num_sms));
            quant_nvfp4_2d_kernel<true><<<grid, 256, 0, s>>>(x, M, K, ldx, mask, scale_src, sa, gs_out, wg, codes, sf);
        } else {
            const int grid = grid_for(tasks, 8, resident_ctas<quant_nvfp4_2d_kernel<false>>(num_sms));
            quant_nvfp4_2d_kernel<false><<<grid, 256, 0, s>>>(x, M, K, ldx, mask, scale_src, sa, gs_out, wg, codes, sf);
        }
        return;
    }
    const int64_t KB = K >> 4;
    if (!row_index && G == 0 && ldx == K && KB >= 4 && (KB & (KB - 1)) == 0) {
        int kb_shift = 0;
        while ((int64_t(1) << kb_shift) < KB) kb_shift++;
        const int64_t nblk = M * KB;
#define BSQ_NVF(R, F, I)                                                                                        \
    launch_dependent(quant_nvfp4_1d_flat_kernel<R, F, I>,                                                      \
                     grid_for(nblk, 2 * 256, resident_ctas<quant_nvfp4_1d_flat_kernel<R, F, I>>(num_sms)), 256, 0, \
                     s, x, nblk, kb_shift, mask, scale_src, sa, gs_out, wg, codes, sf)
        if (nblk < (int64_t(1) << 31)) {
            if (rht) { if (fos) BSQ_NVF(true, true, uint32_t); else BSQ_NVF(true, false, uint32_t); }
            else { if (fos) BSQ_NVF(false, true, uint32_t); else BSQ_NVF(false, false, uint32_t); }
        } else {
            if (rht) { if (fos) BSQ_NVF(true, true, int64_t); else BSQ_NVF(true, false, int64_t); }
            else { if (fos) BSQ_NVF(false, true, int64_t); else BSQ_NVF(false, false, int64_t); }
        }
#undef BSQ_NVF
        return;
    }
    RowMap map{lpr_shift_for(K >> 4)};
    const int grid = grid_for(M, 256 >> map.lpr_shift, num_sms * 8);
    const bool gather = row_index != nullptr, grouped = G > 0;
    const bool i32 = M * K < (int64_t(1) << 31);
#define BSQ_NV1(R, F, GA, GR)                                                                                  \
    do {                                                                                                       \
        if (i32)                                                                                               \
            quant_nvfp4_1d_kernel<R, F, GA, GR, uint32_t><<<grid, 256, 0, s>>>(                                \
                x, M, K, ldx, mask, row_index, G, row_off, sf_off, scale_src, sa, gs_out, wg, codes, sf, map);    \
        else                                                                                                   \
            quant_nvfp4_1d_kernel<R, F, GA, GR, int64_t><<<grid, 256, 0, s>>>(                                 \
                x, M, K, ldx, mask, row_index, G, row_off, sf_off, scale_src, sa, gs_out, wg, codes, sf, map);    \
    } while (0)
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

int launch_quant_nvfp4_fused(const uint16_t *x, int64_t M, int64_t K, bool rht, uint32_t mask, float *gs_out,
                             uint8_t *codes, uint8_t *sf, unsigned int *err, int num_sms, cudaStream_t s) {
    const int64_t KB = K >> 4;
    unsigned int *scratch = reinterpret_cast<unsigned int *>(codes);
    void *args[] = {(void *)&x, (void *)&M, (void *)&K, (void *)&mask, (void *)&scratch,
                    (void *)&gs_out, (void *)&codes, (void *)&sf, (void *)&err};
    const void *kern = rht ? (const void *)quant_nvfp4_fused_kernel<true> : (const void *)quant_nvfp4_fused_kernel<false>;
    const int resident = rht ? resident_ctas<quant_nvfp4_fused_kernel<true>>(num_sms)
                             : resident_ctas<quant_nvfp4_fused_kernel<false>>(num_sms);
    // one resident wave, no more CTAs than 256-block groups of work
    const int grid = grid_for(M * KB, 256, resident);
    return cudaLaunchCooperativeKernel(kern, dim3(grid), dim3(256), args, 0, s) == cudaSuccess ? 0 : 1;
}

// Streaming NVFP4 kernels: CTAs that fit at once (dynamic shared memory
// included), per kernel and device.
template <auto Kern>
static int resident_stream(int num_sms) {
    const int n = g_occupancy.get(
        reinterpret_cast<const void *>(Kern), current_device(),
        [] {
            int v = 0;
            return cudaOccupancyMaxActiveBlocksPerMultiprocessor(&v, Kern, nvs::kThreads, nvs::kSmemBytes) == cudaSuccess
                       ? v
                       : 0;
        },
        [](int v) { return v >= 1; });
    return (n < 1 ? 1 : n) * num_sms;
}

template <int MODE, bool RHT, bool TWO_D>
static int launch_stream_t(const uint16_t *x, int64_t M, int64_t K, uint32_t mask, unsigned int *counter,
                           unsigned int *amax_bits, const float *scale_src, int src_is_amax, float *gs_out,
                           uint8_t *codes, uint8_t *sf, unsigned int *err, int num_sms, cudaStream_t s) {
    auto kern = quant_nvfp4_stream_kernel<MODE, RHT, TWO_D>;
    if (smem_attr_once(reinterpret_cast<const void *>(kern), nvs::kSmemBytes) != BSQ_OK) return 1;
    const int64_t KB = K >> 4;
    const int64_t chunks = TWO_D ? (M >> 4) * ((K + 511) >> 9) : (M * KB + 511) >> 9;
    const int grid = grid_for(chunks, 1, resident_stream<quant_nvfp4_stream_kernel<MODE, RHT, TWO_D>>(num_sms));
    DivU32 div_kb = divu32_for((uint32_t)KB);
    DivU32 div_span = divu32_for((uint32_t)((K + 511) >> 9));
    if (MODE == nvs::FUSED) {
        // one pointer per kernel parameter, in the kernel's order
        void *args[] = {(void *)&x,         (void *)&M,           (void *)&K,      (void *)&div_kb,
                        (void *)&div_span,  (void *)&mask,        (void *)&counter, (void *)&amax_bits,
                        (void *)&scale_src, (void *)&src_is_amax, (void *)&gs_out, (void *)&codes,
                        (void *)&sf,        (void *)&err};
        return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(kern), dim3(grid), dim3(nvs::kThreads), args,
                                           nvs::kSmemBytes, s) == cudaSuccess
                   ? 0
                   : 1;
    }
    if (launch_dependent(kern, grid, nvs::kThreads, nvs::kSmemBytes, s, x, M, K, div_kb, div_span, mask, counter,
                         amax_bits, scale_src, src_is_amax, gs_out, codes, sf, err) != cudaSuccess)
        return 1;
    return cudaGetLastError() == cudaSuccess ? 0 : 1;
}

bool stream_ok(int64_t M, int64_t K, bool block_2d) {
    return K % 64 == 0 && M * (K >> 4) < (int64_t(1) << 32) && (!block_2d || M % 16 == 0);
}

int launch_nvfp4_stream(int mode, const uint16_t *x, int64_t M, int64_t K, bool block_2d, bool rht, uint32_t mask,
                        unsigned int *counter, unsigned int *amax_bits, const float *scale_src, bool src_is_amax,
                        float *gs_out, uint8_t *codes, uint8_t *sf, unsigned int *err, int num_sms, cudaStream_t s) {
    const int sa = src_is_amax ? 1 : 0;
#define BSQ_NVS(MO, R, D)                                                                                        \
    return launch_stream_t<MO, R, D>(x, M, K, mask, counter, amax_bits, scale_src, sa, gs_out, codes, sf, err, \
                                     num_sms, s)
#define BSQ_NVS_RD(MO)                                  \
    do {                                                \
        if (rht) {                                      \
            if (block_2d) BSQ_NVS(MO, true, true);      \
            else BSQ_NVS(MO, true, false);              \
        } else {                                        \
            if (block_2d) BSQ_NVS(MO, false, true);     \
            else BSQ_NVS(MO, false, false);             \
        }                                               \
    } while (0)
    if (mode == nvs::AMAX) BSQ_NVS_RD(nvs::AMAX);
    if (mode == nvs::QUANT) BSQ_NVS_RD(nvs::QUANT);
    BSQ_NVS_RD(nvs::FUSED);
#undef BSQ_NVS_RD
#undef BSQ_NVS
}

void launch_quant_mxfp8(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, bool colwise, bool sr,
                        uint64_t seed, uint32_t stream_id, uint8_t *codes, uint8_t *sf, int num_sms,
                        cudaStream_t s) {
    const PhiloxKeys keys = philox_keys((uint32_t)seed, (uint32_t)(seed >> 32));
    if (!colwise && ldx == K && K % 1024 == 0 && M * (K >> 10) < (int64_t(1) << 31)) {
        const uint32_t nspan = (uint32_t)(M * (K >> 10));
        const DivU32 dspr = divu32_for((uint32_t)(K >> 10));
        if (sr) {
            const int grid = grid_for(nspan, 8, resident_ctas<quant_mxfp8_row_span_kernel<true>>(num_sms));
            quant_mxfp8_row_span_kernel<true><<<grid, 256, 0, s>>>(x, nspan, K, dspr, keys, stream_id, codes, sf);
        } else {
            const int grid = grid_for(nspan, 8, resident_ctas<quant_mxfp8_row_span_kernel<false>>(num_sms));
            quant_mxfp8_row_span_kernel<false><<<grid, 256, 0, s>>>(x, nspan, K, dspr, keys, stream_id, codes, sf);
        }
        return;
    }
    if (!colwise && ldx == K && K % 128 == 0 && M * (K >> 3) < (int64_t(1) << 32)) {
        const int64_t nchunk = M * (K >> 3);
        const DivU32 dk8 = divu32_for((uint32_t)(K >> 3));
        if (sr) {
            const int grid = grid_for(nchunk, 4 * 256, resident_ctas<quant_mxfp8_row_flat_kernel<true>>(num_sms));
            quant_mxfp8_row_flat_kernel<true><<<grid, 256, 0, s>>>(x, nchunk, K, dk8, keys, stream_id, codes, sf);
        } else {
            const int grid = grid_for(nchunk, 4 * 256, resident_ctas<quant_mxfp8_row_flat_kernel<false>>(num_sms));
            quant_mxfp8_row_flat_kernel<false><<<grid, 256, 0, s>>>(x, nchunk, K, dk8, keys, stream_id, codes, sf);
        }
        return;
    }
    if (!colwise) {
        RowMap map{lpr_shift_for(K >> 3)};
        if (map.lpr_shift < 2) map.lpr_shift = 2;  // 4 lanes per block of 32
        const int grid = grid_for(M, 256 >> map.lpr_shift, num_sms * 8);
        const bool i32 = M * ldx < (int64_t(1) << 31);
        if (sr) {
            if (i32) quant_mxfp8_row_kernel<true, uint32_t><<<grid, 256, 0, s>>>(x, M, K, ldx, keys, stream_id, codes, sf, map);
            else quant_mxfp8_row_kernel<true, int64_t><<<grid, 256, 0, s>>>(x, M, K, ldx, keys, stream_id, codes, sf, map);
        } else {
            if (i32) quant_mxfp8_row_kernel<false, uint32_t><<<grid, 256, 0, s>>>(x, M, K, ldx, keys, stream_id, codes, sf, map);
            else quant_mxfp8_row_kernel<false, int64_t><<<grid, 256, 0, s>>>(x, M, K, ldx, keys, stream_id, codes, sf, map);
        }
        return;
    }
    const uint32_t ntile = (uint32_t)((M >> 5) * ((K + 63) >> 6));
    const DivU32 dmt = divu32_for((uint32_t)(M >> 5));
    if (sr) {
#define BSQ_MXC(S, I)                                                                                        \
    quant_mxfp8_col_kernel<S, I><<<grid_for(ntile, 8, resident_ctas<quant_mxfp8_col_kernel<S, I>>(num_sms)), 256, 0, \
                                   s>>>(x, M, K, ldx, ntile, dmt, keys, stream_id, codes, sf)
        if (M * K < (int64_t(1) << 31)) BSQ_MXC(true, uint32_t); else BSQ_MXC(true, int64_t);
    } else {
        if (M * K < (int64_t(1) << 31)) BSQ_MXC(false, uint32_t); else BSQ_MXC(false, int64_t);
#undef BSQ_MXC
    }
}

void launch_requant_transpose(const uint8_t *codes_row, const uint8_t *sf_row, int64_t M, int64_t K, bool sr,
                              uint64_t seed, uint32_t stream_id, uint8_t *codes_col, uint8_t *sf_col,
                              int num_sms, cudaStream_t s) {
    const PhiloxKeys keys = philox_keys((uint32_t)seed, (uint32_t)(seed >> 32));
    const uint32_t ntile = (uint32_t)((M >> 5) * ((K + 63) >> 6));
    const DivU32 dmt = divu32_for((uint32_t)(M >> 5));
#define BSQ_RQT(S, I)                                                                                        \
    requant_transpose_kernel<S, I><<<grid_for(ntile, 8, resident_ctas<requant_transpose_kernel<S, I>>(num_sms)), 256, \
                                     0, s>>>(codes_row, sf_row, M, K, ntile, dmt, keys, stream_id, codes_col, sf_col)
    const bool i32 = M * K < (int64_t(1) << 31);
    if (sr) { if (i32) BSQ_RQT(true, uint32_t); else BSQ_RQT(true, int64_t); }
    else { if (i32) BSQ_RQT(false, uint32_t); else BSQ_RQT(false, int64_t); }
#undef BSQ_RQT
}

void launch_quant_mxfp8_rowcol(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, bool sr, uint64_t seed,
                               uint32_t stream_r, uint32_t stream_c, uint8_t *codes_r, uint8_t *sf_r,
                               uint8_t *codes_c, uint8_t *sf_c, int num_sms, cudaStream_t s) {
    const PhiloxKeys keys = philox_keys((uint32_t)seed, (uint32_t)(seed >> 32));
    const uint32_t ntile = (uint32_t)((M >> 5) * ((K + 63) >> 6));
    const DivU32 dmt = divu32_for((uint32_t)(M >> 5));
#define BSQ_RC(S, I)                                                                                          \
    quant_mxfp8_rowcol_kernel<S, I><<<grid_for(ntile, 8, resident_ctas<quant_mxfp8_rowcol_kernel<S, I>>(num_sms)),  \
                                      256, 0, s>>>(x, M, K, ldx, ntile, dmt, keys, stream_r, stream_c, codes_r, sf_r, \
                                                   codes_c, sf_c)
    const bool i32 = M * K < (int64_t(1) << 31);
    if (sr) { if (i32) BSQ_RC(true, uint32_t); else BSQ_RC(true, int64_t); }
    else { if (i32) BSQ_RC(false, uint32_t); else BSQ_RC(false, int64_t); }
#undef BSQ_RC
}

void launch_requant_nvfp4_mxfp8(const uint8_t *codes_in, const uint8_t *sf_in, const float *gs, int64_t R, int64_t C,
                                bool sr, uint64_t seed, uint32_t stream_id, uint8_t *codes, uint8_t *sf, int num_sms,
                                cudaStream_t s) {
    const PhiloxKeys keys = philox_keys((uint32_t)seed, (uint32_t)(seed >> 32));
    const uint32_t ntile = (uint32_t)((R >> 5) * ((C + 63) >> 6));
    const DivU32 dmt = divu32_for((uint32_t)(R >> 5));
#define BSQ_RQ4(S, I)                                                                                         \
    requant_nvfp4_mxfp8_kernel<S, I><<<grid_for(ntile, 8, resident_ctas<requant_nvfp4_mxfp8_kernel<S, I>>(num_sms)), \
                                       256, 0, s>>>(codes_in, sf_in, gs, R, C, ntile, dmt, keys, stream_id, codes, sf)
    const bool i32 = R * C < (int64_t(1) << 31);
    if (sr) { if (i32) BSQ_RQ4(true, uint32_t); else BSQ_RQ4(true, int64_t); }
    else { if (i32) BSQ_RQ4(false, uint32_t); else BSQ_RQ4(false, int64_t); }
#undef BSQ_RQ4
}

void launch_quant_mxfp4(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, bool sr, uint64_t seed,
                        uint32_t stream_id, uint8_t *codes, uint8_t *sf, int num_sms, cudaStream_t s) {
    const PhiloxKeys keys = philox_keys((uint32_t)seed, (uint32_t)(seed >> 32));
    if (ldx == K && K % 1024 == 0 && M * (K >> 10) < (int64_t(1) << 31)) {
        const uint32_t nspan = (uint32_t)(M * (K >> 10));
        const DivU32 dspr = divu32_for((uint32_t)(K >> 10));
        if (sr) {
            const int grid = grid_for(nspan, 8, resident_ctas<quant_mxfp4_row_span_kernel<true>>(num_sms));
            quant_mxfp4_row_span_kernel<true><<<grid, 256, 0, s>>>(x, nspan, K, dspr, keys, stream_id, codes, sf);
        } else {
            const int grid = grid_for(nspan, 8, resident_ctas<quant_mxfp4_row_span_kernel<false>>(num_sms));
            quant_mxfp4_row_span_kernel<false><<<grid, 256, 0, s>>>(x, nspan, K, dspr, keys, stream_id, codes, sf);
        }
        return;
    }
    RowMap map{lpr_shift_for(K >> 3)};
    if (map.lpr_shift < 2) map.lpr_shift = 2;  // 4 lanes per block of 32
    const int grid = grid_for(M, 256 >> map.lpr_shift, num_sms * 8);
    const bool i32 = M * ldx < (int64_t(1) << 31);
    if (sr) {
        if (i32) quant_mxfp4_row_kernel<true, uint32_t><<<grid, 256, 0, s>>>(x, M, K, ldx, keys, stream_id, codes, sf, map);
        else quant_mxfp4_row_kernel<true, int64_t><<<grid, 256, 0, s>>>(x, M, K, ldx, keys, stream_id, codes, sf, map);
    } else {
        if (i32) quant_mxfp4_row_kernel<false, uint32_t><<<grid, 256, 0, s>>>(x, M, K, ldx, keys, stream_id, codes, sf, map);
        else quant_mxfp4_row_kernel<false, int64_t><<<grid, 256, 0, s>>>(x, M, K, ldx, keys, stream_id, codes, sf, map);
    }
}

void launch_quant_nvfp4_sr(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, bool block_2d, bool rht,
                           uint32_t mask, const int32_t *row_index, const float *scale_src, bool src_is_amax,
                           float *gs_out, bool write_gs, uint64_t seed, uint32_t stream_id, uint8_t *codes,
                           uint8_t *sf, int num_sms, cudaStream_t s) {
    const PhiloxKeys keys = philox_keys((uint32_t)seed, (uint32_t)(seed >> 32));
    const int sa = src_is_amax ? 1 : 0, wg = write_gs ? 1 : 0;
    if (block_2d) {
        const int64_t tasks = (M >> 4) * (((K >> 4) + 7) >> 3);
        if (rht) {
            const int grid = grid_for(tasks, 8, resident_ctas<quant_nvfp4_sr_2d_kernel<true>>(num_sms));
            quant_nvfp4_sr_2d_kernel<true><<<grid, 256, 0, s>>>(x, M, K, ldx, mask, scale_src, sa, gs_out, wg, keys,
                                                                stream_id, codes, sf);
        } else {
            const int grid = grid_for(tasks, 8, resident_ctas<quant_nvfp4_sr_2d_kernel<false>>(num_sms));
            quant_nvfp4_sr_2d_kernel<false><<<grid, 256, 0, s>>>(x, M, K, ldx, mask, scale_src, sa, gs_out, wg, keys,
                                                                 stream_id, codes, sf);
        }
        return;
    }
    RowMap map{lpr_shift_for(K >> 4)};
    const int grid = grid_for(M, 256 >> map.lpr_shift, num_sms * 8);
#define BSQ_NVSR(R, GA, I)                                                                                     \
    quant_nvfp4_sr_1d_kernel<R, GA, I><<<grid, 256, 0, s>>>(x, M, K, ldx, mask, row_index, scale_src, sa, gs_out, wg, \
                                                            keys, stream_id, codes, sf, map)
    // 32-bit offsets within a row and over the output (the source row's start stays 64-bit)
    if (M * K < (int64_t(1) << 31)) {
        if (rht) { if (row_index) BSQ_NVSR(true, true, uint32_t); else BSQ_NVSR(true, false, uint32_t); }
        else { if (row_index) BSQ_NVSR(false, true, uint32_t); else BSQ_NVSR(false, false, uint32_t); }
    } else {
        if (rht) { if (row_index) BSQ_NVSR(true, true, int64_t); else BSQ_NVSR(true, false, int64_t); }
        else { if (row_index) BSQ_NVSR(false, true, int64_t); else BSQ_NVSR(false, false, int64_t); }
    }
#undef BSQ_NVSR
}

void launch_quant_s2f6(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, bool rht, uint32_t mask, int8_t *codes,
                       uint8_t *sf, int num_sms, cudaStream_t s) {
    RowMap map{lpr_shift_for(K >> 4)};
    const int grid = grid_for(M, 256 >> map.lpr_shift, num_sms * 8);
    if (rht) quant_s2f6_kernel<true><<<grid, 256, 0, s>>>(x, M, K, ldx, mask, codes, sf, map);
    else quant_s2f6_kernel<false><<<grid, 256, 0, s>>>(x, M, K, ldx, mask, codes, sf, map);
}

void launch_combine_s2f6(const int8_t *codes, const uint8_t *sf, int64_t K, const int32_t *off, const int32_t *rows,
                         const float *weights, int64_t T, uint32_t mask, uint16_t *out, int64_t ldo, int num_sms,
                         cudaStream_t s) {
    const int grid = grid_for(T * (K >> 4), 256, num_sms * 8);
    combine_s2f6_kernel<<<grid, 256, 0, s>>>(codes, sf, K, off, rows, weights, T, mask, out, ldo);
}

void launch_gather_rows(const void *src, int64_t row_bytes, const int32_t *index, int64_t R, void *dst, int num_sms,
                        cudaStream_t s) {
    const int64_t vec = row_bytes / 16;
    gather_rows_kernel<<<grid_for(R, 8, num_sms * 8), 256, 0, s>>>(static_cast<const uint4 *>(src), vec, index, R,
                                                                    static_cast<uint4 *>(dst));
}

void launch_sf_to_rows(const uint8_t *sf, int64_t rows, int64_t nblk, uint8_t *out, int num_sms, cudaStream_t s) {
    sf_to_rows_kernel<<<grid_for(rows * nblk, 256, num_sms * 8), 256, 0, s>>>(sf, rows, nblk,
                                                                             divu32_for((uint32_t)nblk), out);
}

void launch_sf_from_rows(const uint8_t *in, int64_t rows, int64_t nblk, int G, const int32_t *row_off,
                         const int32_t *sf_off, uint8_t *sf, int num_sms, cudaStream_t s) {
    sf_from_rows_kernel<<<grid_for(rows * nblk, 256, num_sms * 8), 256, 0, s>>>(
        in, rows, nblk, divu32_for((uint32_t)nblk), G, row_off, sf_off, sf);
}

void launch_row_absmax(const uint16_t *x, int64_t T, int64_t K, int64_t ldx, bool rht, uint32_t mask, float *rowmax,
                       int num_sms, cudaStream_t s) {
    const int grid = grid_for(T, 8, num_sms * 8);
    if (rht) row_absmax_kernel<true><<<grid, 256, 0, s>>>(x, T, K, ldx, mask, rowmax);
    else row_absmax_kernel<false><<<grid, 256, 0, s>>>(x, T, K, ldx, mask, rowmax);
}

void launch_gathered_max(const float *rowmax, const int32_t *row_index, int64_t M, unsigned int *amax_bits,
                         unsigned int *counter, float *gs_out, int num_sms, cudaStream_t s) {
    gathered_max_kernel<<<grid_for(M, 256 * 8, num_sms), 256, 0, s>>>(rowmax, row_index, M, amax_bits, counter, gs_out);
}

void launch_gather_sf(const uint8_t *sf_src, int64_t nblk, const int32_t *row_index, int64_t M, int G,
                      const int32_t *row_off, const int32_t *sf_off, uint8_t *sf, int num_sms, cudaStream_t s) {
    // destination rows: M, or with groups at most M + 128 G (each group padded to 128 rows)
    const int64_t ng = ((nblk >> 2) + 3) >> 2;
    const int64_t units = ((M + 128 * (int64_t)G + 127) >> 7) * ng;
    gather_sf_kernel<<<grid_for(units, 2, num_sms * 8), 256, 0, s>>>(sf_src, nblk, divu32_for((uint32_t)ng), row_index,
                                                                      M, G, row_off, sf_off, sf);
}

void launch_rht(const uint16_t *x, uint16_t *y, int64_t M, int64_t K, int64_t ldx, int64_t ldy, uint32_t mask,
                int num_sms, cudaStream_t s) {
    RowMap map{lpr_shift_for(K >> 4)};
    const int grid = grid_for(M, 256 >> map.lpr_shift, num_sms * 8);
    rht_kernel<<<grid, 256, 0, s>>>(x, y, M, K, ldx, ldy, mask, map);
}

}  // namespace bsq
