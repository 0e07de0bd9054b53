// gemm.cu -- block-scaled GEMM for sm_100a: C = alpha * dec(A) dec(B)^T with
// NVFP4 (kind::mxf4nvf4, 16-element E4M3 scales) or MXFP8 (kind::mxf8f6f4,
// 32-element E8M0 scales) operands, both K-major.
//
// Persistent, warp-specialised CTA (10 warps):
//   warp 0      TMA producer: A/B code tiles (128-byte swizzle) and the
//               scale-factor atoms (1-D bulk copies) into a k-stage ring;
//   warp 1      TMEM allocator + MMA issuer: copies the scale atoms an MMA
//               needs to a ring of TMEM slots (tcgen05.cp) right before that
//               MMA, so the copies overlap the previous MMA, issues
//               tcgen05.mma with block scales, commits stage release and
//               accumulator-ready;
//   warps 2..9  epilogue, two warps per TMEM lane quarter (each one half of
//               the tile's columns): tcgen05.ld of the fp32 accumulator,
//               alpha scale, fp32 or bf16 stores (transposed for swap-AB).
// With one 256-column accumulator the epilogue drains TMEM into registers,
// releases it, and stores while the next tile's MMAs run.
// Every mbarrier wait is bounded (device clock); on expiry the CTA records
// a timeout in the error word, drains its own copies, frees TMEM and exits.
// No load uses cluster multicast.
#include <cuda.h>

#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "common.cuh"
#include "devcache.h"
#include "gemm.cuh"
#include "nvfp4.cuh"
#include "sm100.cuh"

namespace bsq {

using namespace sm100;

constexpr uint64_t kTimeoutNs = 2000000000ull;  // 2 s of device time per wait

struct GemmParams {
    const uint8_t *sfA, *sfB;
    const float *gsA, *gsB;
    int64_t MA, NB, K;      // rows of operand A, rows of operand B (per group), K
    int64_t m_lim, n_lim;   // output bounds in operand order (rows of A, rows of B)
    void *C;
    int64_t ldc;
    int64_t sfB_group_bytes;  // bytes between the SF buffers of consecutive groups of B
    int G;
    const int32_t *row_off, *sf_row_off;
    unsigned int *err;
    // NVFP4 output of the quantizing epilogue (pair kernel with QOUT)
    uint8_t *q_codes;     // [rows][NB/2]
    uint8_t *q_sf;        // swizzled, NB/16 blocks per row, rows at the groups' SF offsets
    const float *q_sg;    // the global scale the output is quantized with
    unsigned int *q_amax; // atomicMax of the bits of max |bf16 output| (NULL: not kept)
    int q_fos;            // Four Over Six block scales
    int c_tma;            // skinny bf16 output through shared memory and one TMA tile store
};

template <int FMT>
struct FmtTraits;
template <>
struct FmtTraits<BSQ_NVFP4> {
    static constexpr int kBkElems = 256;     // elements per 128-byte k-tile row
    static constexpr int kMmaK = 64;         // elements per MMA
    static constexpr int kAtomsPerKt = 4;    // 512-byte SF atoms per 128 rows per k-tile
    static constexpr int kVec = 16;
    static constexpr uint32_t kIdescFmt = (1u << 7) | (1u << 10);  // E2M1 x E2M1, UE4M3 scales
};
template <>
struct FmtTraits<BSQ_MXFP4> {
    static constexpr int kBkElems = 256;     // elements per 128-byte k-tile row
    static constexpr int kMmaK = 64;
    static constexpr int kAtomsPerKt = 2;    // 8 blocks of 32 per k-tile: two 4-block atoms
    static constexpr int kVec = 32;
    static constexpr uint32_t kIdescFmt = (1u << 7) | (1u << 10) | (1u << 23);  // E2M1 x E2M1, UE8M0 scales
};
template <>
struct FmtTraits<BSQ_MXFP8> {
    static constexpr int kBkElems = 128;
    static constexpr int kMmaK = 32;
    static constexpr int kAtomsPerKt = 1;
    static constexpr int kVec = 32;
    static constexpr uint32_t kIdescFmt = (0u << 7) | (0u << 10) | (1u << 23);  // E4M3 x E4M3, UE8M0
};

template <int FMT, int BN, int MAXNS = 8>
struct Cfg {
    using T = FmtTraits<FMT>;
    static constexpr int kBM = 128;
    static constexpr int kABytes = 128 * 128;
    static constexpr int kBBytes = BN * 128;
    static constexpr int kNbAtomTiles = (BN + 127) / 128;
    static constexpr int kSfaBytes = T::kAtomsPerKt * 512;
    static constexpr int kSfbBytes = kNbAtomTiles * kSfaBytes;
    static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
    static constexpr int kFit = (220 * 1024) / kStageBytes;
    static constexpr int kStages = kFit > MAXNS ? MAXNS : kFit;
    // skinny (BN = 64) bf16 output staged for one TMA tile store: 64 x 128
    static constexpr int kStagingOff = kStages * kStageBytes;
    static constexpr int kStagingBytes = BN == 64 ? 64 * 128 * 2 : 0;
    static constexpr int kSmemBytes = kStagingOff + kStagingBytes + 1024;  // + alignment slack
    // TMEM scale-factor slots: NVFP4 copies one slot per MMA (4 SFA columns
    // + 4 per 128 rows of B), MXFP8 one slot per k-tile (its atoms cover the
    // 4 MMAs of the k-tile, selected by the scale-factor id)
    // MXFP4 copies one slot per k-tile too, holding both k-atoms (SFA 2 x 4
    // columns, then per 128 rows of B 2 x 4 columns)
    static constexpr int kSlotCols = (FMT == BSQ_MXFP4) ? 8 + 8 * kNbAtomTiles : 4 + 4 * kNbAtomTiles;
    static constexpr int kSlots = (FMT == BSQ_NVFP4) ? 16 : 8;
    static constexpr int kMmaPerKt = T::kBkElems / T::kMmaK;  // 4
    static constexpr int kEpiWarps = 8;
    // two more warps: the scale copiers of the skinny NVFP4 kernel (idle elsewhere)
    static constexpr int kThreads = 32 * (2 + kEpiWarps + 2);
};

// Tile -> (group, m tile, n tile) for the persistent loop.
struct TileInfo {
    int64_t a_row0;   // first operand-A row of the tile (TMA y)
    int64_t sfa_row0; // first SF row of operand A (multiple of 128)
    int64_t m_lim;    // exclusive bound of valid operand-A rows
    int64_t n0;       // first operand-B row inside its group
    int group;
};

template <bool GROUPED>
BSQ_DEV TileInfo tile_info(int64_t t, int64_t m_tiles, const GemmParams &p, const int *tile_start,
                           const int32_t *offs) {
    TileInfo ti;
    if (!GROUPED) {
        ti.a_row0 = (t % m_tiles) * 128;
        ti.sfa_row0 = ti.a_row0;
        ti.m_lim = p.m_lim;
        ti.n0 = t / m_tiles;
        ti.group = 0;
        return ti;
    }
    // largest group g with tile_start[g] <= t (groups without rows own no tile)
    int lo = 0, hi = p.G;
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (tile_start[mid] <= t) lo = mid; else hi = mid;
    }
    const int64_t local = t - tile_start[lo];
    const int64_t mt_g = ((int64_t)offs[lo + 1] - offs[lo] + 127) / 128;  // >= 1 for a group that owns t
    const int64_t mt = local % mt_g;
    ti.a_row0 = (int64_t)offs[lo] + mt * 128;
    ti.sfa_row0 = (int64_t)__ldg(p.sf_row_off + lo) + mt * 128;
    ti.m_lim = min((int64_t)offs[lo + 1], p.m_lim);  // never past the last row of A
    ti.n0 = local / mt_g;
    ti.group = lo;
    return ti;
}

template <int FMT, int BN, int ACC, bool OUT_BF16, bool SWAP, bool GROUPED, int SPLITK = 1>
__global__ void __launch_bounds__(384, SPLITK == 1 ? 1 : 2)
    gemm_bs_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, const GemmParams p) {
    // SPLITK > 1: a cluster of SPLITK CTAs computes one tile, CTA r over the
    // r-th of SPLITK equal runs of k-tiles; the partial sums meet in the
    // rank-0 CTA (distributed shared memory) in rank order.  Three stages
    // (86 KB) and 256 TMEM columns per CTA, so that two CTAs share an SM.
    static_assert(SPLITK == 1 || (SWAP && BN == 64 && !GROUPED), "split-K: the skinny swap-AB tile only");
    using C_ = Cfg<FMT, BN, SPLITK == 1 ? 8 : 3>;
    constexpr int kTmemCols = SPLITK == 1 ? 512 : 256;
    using T = typename C_::T;
    constexpr int NS = C_::kStages;
    // Skinny NVFP4 (swap-AB): the tiny MMAs leave the MMA thread bound by its
    // own tcgen05 issue (8 scale copies + 4 MMAs + a commit per k-tile), so two
    // copier threads (warps 10 and 11) copy the SFA and SFB atoms of each
    // stage into that stage's own TMEM slots and commit to sfa_bar / sfb_bar;
    // the MMA thread issues only MMAs.  A stage's slots are free whenever its
    // smem is: the producer refills a stage only after its MMAs completed.
    constexpr bool COPIERS = FMT == BSQ_NVFP4 && SWAP;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[NS], empty_bar[NS], accf_bar[ACC], acce_bar[ACC], drain_bar;
    __shared__ __align__(8) uint64_t sfa_bar[COPIERS ? NS : 1], sfb_bar[COPIERS ? NS : 1];
    __shared__ __align__(8) uint64_t stg_full, stg_free;  // skinny bf16 output staging (p.c_tma)
    __shared__ uint32_t tmem_base_slot;
    __shared__ volatile int abort_flag;
    __shared__ int tile_start[GROUPED ? 1025 : 1];
    __shared__ int32_t offs[GROUPED ? 1025 : 1];

    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = sA + NS * C_::kABytes;
    uint8_t *sSFA = sB + NS * C_::kBBytes;
    uint8_t *sSFB = sSFA + NS * C_::kSfaBytes;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t m_tiles = (p.MA + 127) / 128;
    const int64_t n_tiles = (p.NB + BN - 1) / BN;
    const int64_t k_tiles = (p.K + T::kBkElems - 1) / T::kBkElems;
    const int64_t KBT = p.K / (T::kVec * 4);  // SF atoms per 128-row tile along K

    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; i++) {
            mbar_init(smem_u32(&full_bar[i]), 1);
            mbar_init(smem_u32(&empty_bar[i]), 1);
        }
        for (int i = 0; i < ACC; i++) {
            mbar_init(smem_u32(&accf_bar[i]), 1);
            mbar_init(smem_u32(&acce_bar[i]), C_::kEpiWarps);
        }
        mbar_init(smem_u32(&drain_bar), 1);
        mbar_init(smem_u32(&stg_full), C_::kEpiWarps);
        mbar_init(smem_u32(&stg_free), 1);
        if (COPIERS)
            for (int i = 0; i < NS; i++) {
                mbar_init(smem_u32(&sfa_bar[i]), 1);
                mbar_init(smem_u32(&sfb_bar[i]), 1);
            }
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&tmem_base_slot), kTmemCols);
        tmem_relinquish();
    }
    // The set-up above touches no global memory, so it overlaps the previous
    // kernel under launch overlap; from here on the previous kernel has
    // completed and its writes are visible.
    grid_dependency_wait();
    grid_dependents_launch();
    // grouped: per-group tile prefix (one warp, 32 groups per step)
    int64_t total_tiles = m_tiles * n_tiles;
    if (GROUPED) {
        if (warp == 2) {
            for (int i = lane; i <= p.G; i += 32) offs[i] = __ldg(p.row_off + i);
            __syncwarp();
            int carry = 0;
            for (int g0 = 0; g0 < p.G; g0 += 32) {
                int g = g0 + lane;
                int cnt = 0;
                if (g < p.G) {
                    int rows = offs[g + 1] - offs[g];
                    cnt = ((rows + 127) / 128) * (int)n_tiles;
                }
                int incl = cnt;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                    if (lane >= o) incl += v;
                }
                if (g < p.G) tile_start[g] = carry + incl - cnt;
                carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
            }
            if (lane == 0) tile_start[p.G] = carry;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_slot;
    if (GROUPED) total_tiles = tile_start[p.G];

    constexpr int SF_TMEM0 = ACC * BN;  // first TMEM column of the scale-factor slots
    static_assert(ACC * BN + C_::kSlots * C_::kSlotCols <= kTmemCols, "TMEM budget");
    static_assert(!COPIERS || ACC * BN + NS * C_::kMmaPerKt * C_::kSlotCols <= kTmemCols, "TMEM budget (copiers)");
    // this CTA's tiles and k-tiles (split-K: one tile per cluster, launched as
    // tiles x SPLITK CTAs)
    const uint32_t crank = SPLITK > 1 ? cluster_ctarank() : 0u;
    const int64_t t_first = blockIdx.x / SPLITK, t_step = gridDim.x / SPLITK;
    const int64_t kt_begin = k_tiles * crank / SPLITK, kt_end = k_tiles * (crank + 1) / SPLITK;

    // split-K: what an epilogue thread carries from its drain to the reduction
    bool sk_have = false;
    int64_t sk_a_row0 = 0, sk_m_lim = 0, sk_n0 = 0;
    float sk_alpha = 1.0f;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0, armed = 0, armed_par = 0;
            bool ok = true;
            for (int64_t t = t_first; t < total_tiles && ok; t += t_step) {
                TileInfo ti = tile_info<GROUPED>(t, m_tiles, p, tile_start, offs);
                const int64_t nb0 = ti.n0 * BN;
                const int64_t b_row0 = (int64_t)ti.group * p.NB + nb0;
                const uint8_t *sfa_tile = p.sfA + (ti.sfa_row0 / 128) * KBT * 512;
                const uint8_t *sfb_base = p.sfB + (int64_t)ti.group * p.sfB_group_bytes;
                for (int64_t kt = kt_begin; kt < kt_end; kt++) {
                    if (!mbar_wait(smem_u32(&empty_bar[s]), ph ^ 1u, &abort_flag, p.err, 1, kTimeoutNs)) {
                        ok = false;
                        break;
                    }
                    const int64_t krem = p.K - kt * T::kBkElems;
                    const int nmma = krem >= T::kBkElems ? C_::kMmaPerKt : (int)(krem / T::kMmaK);
                    const int atoms = (FMT == BSQ_NVFP4) ? nmma : (FMT == BSQ_MXFP4) ? (nmma + 1) / 2 : 1;
                    uint32_t bytes = C_::kABytes + C_::kBBytes + atoms * 512;
                    int nbat = 0;
                    for (int r = 0; r < C_::kNbAtomTiles; r++)
                        if (nb0 + 128 * r < p.NB) nbat++;
                    bytes += nbat * atoms * 512;
                    const uint32_t fb = smem_u32(&full_bar[s]);
                    mbar_arrive_expect_tx(fb, bytes);
                    tma_load_2d(smem_u32(sA + s * C_::kABytes), &tmA, fb, (int32_t)(kt * 128), (int32_t)ti.a_row0);
                    tma_load_2d(smem_u32(sB + s * C_::kBBytes), &tmB, fb, (int32_t)(kt * 128), (int32_t)b_row0);
                    bulk_load(smem_u32(sSFA + s * C_::kSfaBytes), sfa_tile + kt * C_::kSfaBytes, atoms * 512, fb);
                    for (int r = 0; r < nbat; r++)
                        bulk_load(smem_u32(sSFB + s * C_::kSfbBytes + r * C_::kSfaBytes),
                                  sfb_base + ((nb0 / 128 + r) * KBT) * 512 + kt * C_::kSfaBytes, atoms * 512, fb);
                    armed |= 1u << s;
                    armed_par = (armed_par & ~(1u << s)) | (ph << s);
                    if (++s == NS) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            // drain: every armed stage's latest phase must have landed before exit
            for (int i = 0; i < NS; i++)
                if (armed & (1u << i)) {
                    volatile int never = 0;
                    mbar_wait(smem_u32(&full_bar[i]), (armed_par >> i) & 1u, &never, p.err, 2, kTimeoutNs);
                }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // One thread issues every tcgen05 op, so its own instruction count
        // bounds the MMA rate: descriptors are kept as 32-bit words and
        // stepped with adds, the per-MMA offsets are compile-time constants.
        if (lane == 0) {
            const uint32_t idesc = T::kIdescFmt | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
            constexpr uint32_t kOpHi = smem_desc_hi(1024, 2);  // K-major, 128-byte swizzle, 8-row groups 1 KB apart
            constexpr uint32_t kSfHi = smem_desc_hi(128, 0);   // scale atoms: 32 rows of 16 bytes
            const uint32_t a_lo0 = smem_desc_lo(smem_u32(sA), 16), b_lo0 = smem_desc_lo(smem_u32(sB), 16);
            const uint32_t sfa_lo0 = smem_desc_lo(smem_u32(sSFA), 0), sfb_lo0 = smem_desc_lo(smem_u32(sSFB), 0);
            const uint32_t sf_t0 = tmem_base + SF_TMEM0;
            constexpr uint32_t kSfAtomLo = 512 >> 4;                // one atom, in descriptor units
            constexpr uint32_t kSfbTileLo = C_::kSfaBytes >> 4;    // next 128 rows of B
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            bool issued = false;
            uint32_t ktc = 0;  // k-tiles issued: selects the scale slots
            int64_t it = 0;
            for (int64_t t = t_first; t < total_tiles && ok; t += t_step, it++) {
                const int a = (int)(it % ACC);
                const uint32_t aph = (uint32_t)((it / ACC) & 1);
                if (!mbar_wait(smem_u32(&acce_bar[a]), aph ^ 1u, &abort_flag, p.err, 3, kTimeoutNs)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(a * BN);
                // 32-bit k-tile bookkeeping (on the MMA thread's critical path)
                const uint32_t kt_lo = (uint32_t)kt_begin, kt_hi = (uint32_t)kt_end;
                const uint32_t kt_full = (uint32_t)(p.K / T::kBkElems);
                const int nmma_tail = (int)((p.K % T::kBkElems) / T::kMmaK);
                for (uint32_t kt = kt_lo; kt < kt_hi; kt++, ktc++) {
                    if (!mbar_test_wait(smem_u32(&full_bar[s]), ph) &&
                        !mbar_wait(smem_u32(&full_bar[s]), ph, &abort_flag, p.err, 4, kTimeoutNs)) {
                        ok = false;
                        break;
                    }
                    if constexpr (COPIERS) {  // this stage's scale atoms are in its TMEM slots
                        if (!(mbar_test_wait(smem_u32(&sfa_bar[s]), ph) ||
                              mbar_wait(smem_u32(&sfa_bar[s]), ph, &abort_flag, p.err, 9, kTimeoutNs)) ||
                            !(mbar_test_wait(smem_u32(&sfb_bar[s]), ph) ||
                              mbar_wait(smem_u32(&sfb_bar[s]), ph, &abort_flag, p.err, 10, kTimeoutNs))) {
                            ok = false;
                            break;
                        }
                    }
                    tc_fence_after();
                    const uint32_t a_lo = a_lo0 + (uint32_t)s * (C_::kABytes >> 4);
                    const uint32_t b_lo = b_lo0 + (uint32_t)s * (C_::kBBytes >> 4);
                    const uint32_t sfa_lo = sfa_lo0 + (uint32_t)s * (C_::kSfaBytes >> 4);
                    const uint32_t sfb_lo = sfb_lo0 + (uint32_t)s * (C_::kSfbBytes >> 4);
                    const bool full_kt = kt < kt_full;
                    const int nmma = full_kt ? C_::kMmaPerKt : nmma_tail;
                    if (FMT == BSQ_NVFP4) {
                        // four slots per k-tile, one per MMA: its SFA atom, then one atom per 128 rows of B
                        // (with copiers: the stage's own slots, already filled)
                        const uint32_t slot0 = COPIERS ? sf_t0 + (uint32_t)s * (4 * C_::kSlotCols)
                                                       : sf_t0 + (ktc & (C_::kSlots / 4 - 1)) * (4 * C_::kSlotCols);
                        auto issue = [&](int j) {
                            const uint32_t slot = slot0 + (uint32_t)j * C_::kSlotCols;
                            if constexpr (!COPIERS) {
                                tmem_cp_sf_atom(slot, desc_pack(sfa_lo + kSfAtomLo * j, kSfHi));
#pragma unroll
                                for (int r = 0; r < C_::kNbAtomTiles; r++)
                                    tmem_cp_sf_atom(slot + 4 + 4 * r,
                                                    desc_pack(sfb_lo + kSfbTileLo * r + kSfAtomLo * j, kSfHi));
                            }
                            mma_nvfp4(d_tmem, desc_pack(a_lo + 2 * j, kOpHi), desc_pack(b_lo + 2 * j, kOpHi), idesc, slot,
                                      slot + 4, (kt > kt_lo || j > 0) ? 1u : 0u);
                        };
                        if (full_kt) {
#pragma unroll
                            for (int j = 0; j < C_::kMmaPerKt; j++) issue(j);
                        } else {
                            for (int j = 0; j < nmma; j++) issue(j);
                        }
                    } else if (FMT == BSQ_MXFP4) {
                        // one slot per k-tile: SFA k-atom a at columns 4a, SFB k-atom a (all
                        // 128-row tiles of B, contiguous) at 8 + 4 kNbAtomTiles a; MMA j reads
                        // k-atom j / 2, scale bytes 2 (j % 2) and 2 (j % 2) + 1 (id 2 (j % 2))
                        const uint32_t slot = sf_t0 + (ktc & (C_::kSlots - 1)) * C_::kSlotCols;
                        constexpr uint32_t kSfb0 = 8, kSfbA = 4 * C_::kNbAtomTiles;
                        const int natoms = (nmma + 1) / 2;
                        for (int a = 0; a < natoms; a++) {
                            tmem_cp_sf_atom(slot + 4 * a, desc_pack(sfa_lo + kSfAtomLo * a, kSfHi));
#pragma unroll
                            for (int r = 0; r < C_::kNbAtomTiles; r++)
                                tmem_cp_sf_atom(slot + kSfb0 + kSfbA * a + 4 * r,
                                                desc_pack(sfb_lo + kSfbTileLo * r + kSfAtomLo * a, kSfHi));
                        }
                        auto issue = [&](int j) {
                            const uint32_t id = 2u * (uint32_t)(j & 1), a = (uint32_t)(j >> 1);
                            mma_mxfp4(d_tmem, desc_pack(a_lo + 2 * j, kOpHi), desc_pack(b_lo + 2 * j, kOpHi),
                                      idesc | (id << 29) | (id << 4), (slot + 4 * a) | (id << 30),
                                      (slot + kSfb0 + kSfbA * a) | (id << 30), (kt > kt_lo || j > 0) ? 1u : 0u);
                        };
                        if (full_kt) {
#pragma unroll
                            for (int j = 0; j < C_::kMmaPerKt; j++) issue(j);
                        } else {
                            for (int j = 0; j < nmma; j++) issue(j);
                        }
                    } else {
                        // one slot per k-tile: its atoms cover the 4 MMAs, selected by the scale-factor id
                        const uint32_t slot = sf_t0 + (ktc & (C_::kSlots - 1)) * C_::kSlotCols;
                        tmem_cp_sf_atom(slot, desc_pack(sfa_lo, kSfHi));
#pragma unroll
                        for (int r = 0; r < C_::kNbAtomTiles; r++)
                            tmem_cp_sf_atom(slot + 4 + 4 * r, desc_pack(sfb_lo + kSfbTileLo * r, kSfHi));
                        // scale byte j of each 32-bit SF column: in the descriptor and in
                        // the top bits of the TMEM scale address
                        auto issue = [&](int j) {
                            mma_mxfp8(d_tmem, desc_pack(a_lo + 2 * j, kOpHi), desc_pack(b_lo + 2 * j, kOpHi),
                                      idesc | ((uint32_t)j << 29) | ((uint32_t)j << 4), slot | ((uint32_t)j << 30),
                                      (slot + 4) | ((uint32_t)j << 30), (kt > kt_lo || j > 0) ? 1u : 0u);
                        };
                        if (full_kt) {
#pragma unroll
                            for (int j = 0; j < C_::kMmaPerKt; j++) issue(j);
                        } else {
                            for (int j = 0; j < nmma; j++) issue(j);
                        }
                    }
                    issued = true;
                    tc_commit(smem_u32(&empty_bar[s]));
                    if (++s == NS) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit(smem_u32(&accf_bar[a]));
            }
            if (issued) {
                // all MMAs issued by this CTA have finished before TMEM is freed
                tc_commit(smem_u32(&drain_bar));
                volatile int never = 0;
                mbar_wait(smem_u32(&drain_bar), 0, &never, p.err, 5, kTimeoutNs);
            }
        }
    } else if (warp < 2 + C_::kEpiWarps) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;             // TMEM lane quarter this warp may access
        const int half = (warp - 2) >> 2;   // which half of the tile's columns
        constexpr int HC = BN / 2;          // columns per warp
        const int row = 32 * q + lane;
        int64_t it = 0;
        for (int64_t t = t_first; t < total_tiles; t += t_step, it++) {
            TileInfo ti = tile_info<GROUPED>(t, m_tiles, p, tile_start, offs);
            const int a = (int)(it % ACC);
            const uint32_t aph = (uint32_t)((it / ACC) & 1);
            float alpha = 1.0f;  // read before the wait: off the drain's critical path
            if (FMT == BSQ_NVFP4) {
                const float ga = p.gsA ? __ldg(p.gsA) : 1.0f;
                const float gb = p.gsB ? __ldg(p.gsB + ti.group) : 1.0f;
                alpha = __fmul_rn(ga, gb);
            }
            if (!mbar_wait(smem_u32(&accf_bar[a]), aph, &abort_flag, p.err, 6, kTimeoutNs)) break;
            tc_fence_after();
            const int64_t ar = ti.a_row0 + row;           // operand-A row of this thread
            const bool row_ok = ar < ti.m_lim;
            const int64_t nb0 = ti.n0 * BN + half * HC;   // first column of this warp
            const int64_t n_lim = p.n_lim;
            const uint32_t tbase = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * BN + half * HC);
            if constexpr (SPLITK > 1) {
                // this CTA's partial sums (HC = 32 columns of one row) into its
                // shared memory, column-major [64][128]: the stages are no longer read
                uint32_t part[32];
                if (kt_begin < kt_end) {
                    tmem_ld32(tbase, part);
                    tmem_ld_wait();
                    tc_fence_before();
                } else {
#pragma unroll
                    for (int c = 0; c < 32; c++) part[c] = 0u;  // no k-tile in this CTA's run
                }
                float *red = reinterpret_cast<float *>(sA);
#pragma unroll
                for (int c = 0; c < 32; c++) red[(half * HC + c) * 128 + row] = __uint_as_float(part[c]);
                sk_have = true;
                sk_a_row0 = ti.a_row0;
                sk_m_lim = ti.m_lim;
                sk_n0 = ti.n0 * BN;
                sk_alpha = alpha;
                (void)row_ok;
                (void)nb0;
                (void)n_lim;
                continue;
            } else if (SWAP && OUT_BF16 && SPLITK == 1 && p.c_tma) {
                // the tile as bf16 into the staging buffer [64 tokens][128 W rows],
                // written out by one TMA tile store (clipped at C's edges)
                uint32_t r[32];
                tmem_ld32(tbase, r);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&acce_bar[a]));
                // the previous tile's store has finished reading the buffer
                if (it > 0 &&
                    !mbar_wait(smem_u32(&stg_free), (uint32_t)((it - 1) & 1), &abort_flag, p.err, 13, kTimeoutNs))
                    break;
                uint16_t *stg = reinterpret_cast<uint16_t *>(smem + C_::kStagingOff);
#pragma unroll
                for (int j = 0; j < 32; j++) {
                    const __nv_bfloat16 h = __float2bfloat16_rn(__fmul_rn(alpha, __uint_as_float(r[j])));
                    stg[(half * HC + j) * 128 + row] = *reinterpret_cast<const uint16_t *>(&h);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&stg_full));
                if (threadIdx.x == 64) {
                    if (mbar_wait(smem_u32(&stg_full), (uint32_t)(it & 1), &abort_flag, p.err, 14, kTimeoutNs)) {
                        tma_store_2d(&tmC, smem_u32(stg), (int32_t)ti.a_row0, (int32_t)(ti.n0 * BN));
                        bulk_commit();
                        bulk_wait_read<0>();
                    }
                    mbar_arrive(smem_u32(&stg_free));
                }
                (void)row_ok;
                (void)nb0;
                (void)n_lim;
                continue;
            } else if (OUT_BF16 && ACC == 1) {
                // drain this warp's columns into registers (two loads per wait),
                // release the accumulator, then store
                uint32_t pk[HC / 2];
#pragma unroll
                for (int c = 0; c < HC / 32; c += 2) {
                    uint32_t r0[32], r1[32];
                    tmem_ld32(tbase + 32 * c, r0);
                    tmem_ld32(tbase + 32 * (c + 1), r1);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 16; j++) {
                        __nv_bfloat162 h0 = __floats2bfloat162_rn(__fmul_rn(alpha, __uint_as_float(r0[2 * j])),
                                                                  __fmul_rn(alpha, __uint_as_float(r0[2 * j + 1])));
                        __nv_bfloat162 h1 = __floats2bfloat162_rn(__fmul_rn(alpha, __uint_as_float(r1[2 * j])),
                                                                  __fmul_rn(alpha, __uint_as_float(r1[2 * j + 1])));
                        pk[16 * c + j] = *reinterpret_cast<uint32_t *>(&h0);
                        pk[16 * (c + 1) + j] = *reinterpret_cast<uint32_t *>(&h1);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&acce_bar[a]));
                if (!row_ok) continue;
#pragma unroll
                for (int c = 0; c < HC / 32; c++) {
                    const int64_t n = nb0 + 32 * c;
                    if (!SWAP) {
                        __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.C) + ar * p.ldc + n;
                        if (n + 32 <= n_lim) {
                            uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
                            for (int v = 0; v < 4; v++)
                                d4[v] = make_uint4(pk[16 * c + 4 * v], pk[16 * c + 4 * v + 1], pk[16 * c + 4 * v + 2],
                                                   pk[16 * c + 4 * v + 3]);
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; j++)
                                if (n + j < n_lim) {
                                    uint32_t w = pk[16 * c + j / 2];
                                    uint16_t h = (j & 1) ? (uint16_t)(w >> 16) : (uint16_t)(w & 0xFFFFu);
                                    reinterpret_cast<uint16_t *>(dst)[j] = h;
                                }
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; j++)
                            if (n + j < n_lim) {
                                uint32_t w = pk[16 * c + j / 2];
                                uint16_t h = (j & 1) ? (uint16_t)(w >> 16) : (uint16_t)(w & 0xFFFFu);
                                reinterpret_cast<uint16_t *>(p.C)[(n + j) * p.ldc + ar] = h;
                            }
                    }
                }
            } else {
#pragma unroll 1
                for (int c = 0; c < HC / 32; c++) {
                    uint32_t r[32];
                    tmem_ld32(tbase + 32 * c, r);
                    tmem_ld_wait();
                    if (c == HC / 32 - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(smem_u32(&acce_bar[a]));
                    }
                    if (!row_ok) continue;
                    const int64_t n = nb0 + 32 * c;
                    float v[32];
#pragma unroll
                    for (int j = 0; j < 32; j++) v[j] = __fmul_rn(alpha, __uint_as_float(r[j]));
                    if (!SWAP) {
                        if (OUT_BF16) {
                            __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.C) + ar * p.ldc + n;
                            if (n + 32 <= n_lim) {
                                uint32_t w[16];
#pragma unroll
                                for (int j = 0; j < 16; j++) {
                                    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
                                    w[j] = *reinterpret_cast<uint32_t *>(&h);
                                }
                                uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
                                for (int x = 0; x < 4; x++) d4[x] = make_uint4(w[4 * x], w[4 * x + 1], w[4 * x + 2], w[4 * x + 3]);
                            } else {
                                for (int j = 0; j < 32; j++)
                                    if (n + j < n_lim) dst[j] = __float2bfloat16_rn(v[j]);
                            }
                        } else {
                            float *dst = static_cast<float *>(p.C) + ar * p.ldc + n;
                            if (n + 32 <= n_lim) {
                                float4 *d4 = reinterpret_cast<float4 *>(dst);
#pragma unroll
                                for (int x = 0; x < 8; x++) d4[x] = make_float4(v[4 * x], v[4 * x + 1], v[4 * x + 2], v[4 * x + 3]);
                            } else {
                                for (int j = 0; j < 32; j++)
                                    if (n + j < n_lim) dst[j] = v[j];
                            }
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; j++)
                            if (n + j < n_lim) {
                                if (OUT_BF16)
                                    static_cast<__nv_bfloat16 *>(p.C)[(n + j) * p.ldc + ar] = __float2bfloat16_rn(v[j]);
                                else
                                    static_cast<float *>(p.C)[(n + j) * p.ldc + ar] = v[j];
                            }
                    }
                }
            }
        }
        // every TMA store of the staged tiles has completed before the CTA exits
        if (SWAP && OUT_BF16 && SPLITK == 1 && p.c_tma && threadIdx.x == 64) bulk_wait<0>();
    } else if constexpr (COPIERS) {
        // ------------------------------------------------------------ scale copiers
        // warp 10: SFA atoms, warp 11: SFB atoms; each walks the same tiles and
        // k-tiles as the MMA thread, waits for the stage's data, copies the
        // atoms of its MMAs into the stage's slots and commits to its barrier
        if (lane == 0) {
            const bool sfa_side = warp == 2 + C_::kEpiWarps;
            constexpr uint32_t kSfHi = smem_desc_hi(128, 0);   // scale atoms: 32 rows of 16 bytes
            constexpr uint32_t kSfAtomLo = 512 >> 4;
            constexpr uint32_t kSfbTileLo = C_::kSfaBytes >> 4;
            const uint32_t sfa_lo0 = smem_desc_lo(smem_u32(sSFA), 0), sfb_lo0 = smem_desc_lo(smem_u32(sSFB), 0);
            const uint32_t sf_t0 = tmem_base + SF_TMEM0;
            uint64_t *bars = sfa_side ? sfa_bar : sfb_bar;
            int s = 0;
            uint32_t ph = 0;
            int last = -1;
            uint32_t last_ph = 0;
            bool ok = true;
            for (int64_t t = t_first; t < total_tiles && ok; t += t_step) {
                for (int64_t kt = kt_begin; kt < kt_end; kt++) {
                    if (!mbar_test_wait(smem_u32(&full_bar[s]), ph) &&
                        !mbar_wait(smem_u32(&full_bar[s]), ph, &abort_flag, p.err, 11, kTimeoutNs)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int64_t krem = p.K - kt * T::kBkElems;
                    const int nmma = krem >= T::kBkElems ? C_::kMmaPerKt : (int)(krem / T::kMmaK);
                    const uint32_t slot0 = sf_t0 + (uint32_t)s * (4 * C_::kSlotCols);
                    if (sfa_side) {
                        const uint32_t lo = sfa_lo0 + (uint32_t)s * (C_::kSfaBytes >> 4);
                        for (int j = 0; j < nmma; j++)
                            tmem_cp_sf_atom(slot0 + (uint32_t)j * C_::kSlotCols, desc_pack(lo + kSfAtomLo * j, kSfHi));
                    } else {
                        const uint32_t lo = sfb_lo0 + (uint32_t)s * (C_::kSfbBytes >> 4);
                        for (int j = 0; j < nmma; j++)
#pragma unroll
                            for (int r = 0; r < C_::kNbAtomTiles; r++)
                                tmem_cp_sf_atom(slot0 + (uint32_t)j * C_::kSlotCols + 4 + 4 * r,
                                                desc_pack(lo + kSfbTileLo * r + kSfAtomLo * j, kSfHi));
                    }
                    tc_commit(smem_u32(&bars[s]));
                    last = s;
                    last_ph = ph;
                    if (++s == NS) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            // this thread's copies have executed before the CTA frees TMEM
            if (last >= 0) {
                volatile int never = 0;
                mbar_wait(smem_u32(&bars[last]), last_ph, &never, p.err, 12, kTimeoutNs);
            }
        }
    }
    if constexpr (SPLITK > 1) {
        // every thread of the cluster passes both barriers: the partials are
        // in shared memory after the first, read by rank 0 before the second
        __syncthreads();
        cluster_sync();
        if (sk_have) {
            // CTA r reduces rows [r R, r R + R) of the tile, R = 128 / SPLITK:
            // element e of its slice is column e / R, row r R + e % R (consecutive
            // threads on consecutive rows: conflict-free shared reads, adjacent
            // output addresses).  Each thread's 32 / SPLITK elements: all
            // 32 partials are loaded first (independent remote loads in flight
            // together), then added in rank order 0, 1, ...
            constexpr int R = 128 / SPLITK, PER = 32 / SPLITK;
            const int t = threadIdx.x - 64;  // the 256 epilogue threads
            const uint32_t red0 = smem_u32(sA);
            uint32_t base[SPLITK];
#pragma unroll
            for (int r = 0; r < SPLITK; r++) base[r] = mapa(red0, (uint32_t)r);
            float v[SPLITK][PER];
#pragma unroll
            for (int i = 0; i < PER; i++) {
                const int e = t + 256 * i, col = e / R, row = (int)crank * R + e % R;
#pragma unroll
                for (int r = 0; r < SPLITK; r++) v[r][i] = ld_shared_cluster_f32_nv(base[r] + 4u * (uint32_t)(col * 128 + row));
            }
            const int64_t n_lim = p.n_lim;
#pragma unroll
            for (int i = 0; i < PER; i++) {
                const int e = t + 256 * i, col = e / R, row = (int)crank * R + e % R;
                float sum = v[0][i];
#pragma unroll
                for (int r = 1; r < SPLITK; r++) sum = __fadd_rn(sum, v[r][i]);
                const int64_t ar = sk_a_row0 + row, n = sk_n0 + col;
                if (ar < sk_m_lim && n < n_lim) {
                    const float y = __fmul_rn(sk_alpha, sum);
                    if (OUT_BF16) static_cast<__nv_bfloat16 *>(p.C)[n * p.ldc + ar] = __float2bfloat16_rn(y);
                    else static_cast<float *>(p.C)[n * p.ldc + ar] = y;
                }
            }
        }
        __syncthreads();
        cluster_sync();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ============================================================ CTA-pair kernel
// Two CTAs of a cluster compute one 256x256 tile with tcgen05 cta_group::2:
// CTA r loads rows [128r, 128r+128) of the A tile and of the B tile (the
// MMA reads B across the pair), plus the scale factors its half needs (its
// own 128 SFA rows, all 256 SFB rows).  Per FLOP this moves a third fewer
// bytes from L2 than a 128x256 single-CTA tile.  No load uses multicast.
//
// Warp roles (14 warps per CTA):
//   0        producer: A/B tiles with pair TMA (completion on the leader's
//            full barrier), this CTA's scale tiles with plain TMA (its own
//            sf_full barrier);
//   1        TMEM allocator; in the leader, lane 0 issues the MMAs.  It only
//            waits on mbarriers and issues MMAs and commits;
//   2..5     scale warps, one per TMEM lane quarter: read the stage's scale
//            atoms from shared memory and write them into the stage's TMEM
//            scale slots with tcgen05.st (SFB replicated into every quarter,
//            SFA only in the column each quarter reads), then arrive on the
//            leader's sf_ready barrier (both CTAs; except with the quantizing
//            epilogue, the leader's warps first wait for the stage's A/B
//            halves, so that sf_ready is the MMA thread's only wait per
//            k-tile).  No tcgen05.cp is used:
//            copies execute in the tensor pipe between the MMAs, TMEM stores
//            from other warps do not;
//   6..13    epilogue, two warps per lane quarter (one half of the 256
//            columns each): tcgen05.ld of the accumulator, alpha, bf16/fp32,
//            staged through shared memory (32-row boxes, 64-byte swizzle) and
//            written with TMA tile stores; boxes that cross a group's last
//            row use per-thread stores instead.  bf16 tiles are drained into
//            registers and the accumulator released before the stores, which
//            go through two boxes per warp (14 warps leave 128 registers per
//            thread; the shared memory left over holds five stages).
// Hand-overs across the pair use relaxed cluster-scope arrives: the TMEM
// stores (scales) or loads (accumulator) they announce have completed
// (tcgen05.wait) and are ordered by tcgen05 fences before the arrive.
// TMEM: columns 0..255 accumulator, then per stage the SFB slot (NVFP4: 4
// MMAs x 2 atoms x 4 columns) and the SFA slot (4 MMAs x 4 columns).
template <int FMT, bool GROUPED>
struct Cfg2 {
    using T = FmtTraits<FMT>;
    static constexpr int kABytes = 128 * 128;
    static constexpr int kBBytes = 128 * 128;  // this CTA's half of the 256-row B tile
    static constexpr int kSfaBytes = T::kAtomsPerKt * 512;
    static constexpr int kSfbBytes = 2 * kSfaBytes;
    static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
    static constexpr int kEpiWarps = 8;
    static constexpr int kSfWarps = 4;
    static constexpr int kThreads = 32 * (2 + kSfWarps + kEpiWarps);
    static constexpr int kBoxBytes = 2048;                          // 32 rows x 64 bytes
    static constexpr int kBoxes = 2;                                // per epilogue warp: double-buffered
    static constexpr int kStagingBytes = kEpiWarps * kBoxes * kBoxBytes;
    static constexpr int kSmemLimit = 232448;                       // 227 KB per CTA
    static constexpr int kStaticEst = GROUPED ? 9728 : 512;   // grouped: offsets, tile starts, NVFP4 tables
    static constexpr int kFit = (kSmemLimit - 2048 - kStagingBytes - kStaticEst) / kStageBytes;
    static constexpr int kStages = kFit > 5 ? 5 : kFit;             // TMEM holds up to 5 stages of scales
    static constexpr int kStagingOff = (kStages * kStageBytes + 1023) / 1024 * 1024;
    static constexpr int kSmemBytes = kStagingOff + kStagingBytes + 1024;
    static constexpr int kMmaPerKt = T::kBkElems / T::kMmaK;
    // TMEM scale slots of stage s: SFB at kSfb0 + kSfbCols*s, SFA at kSfa0 + kSfaCols*s
    static constexpr int kSfbCols = (FMT == BSQ_NVFP4) ? 32 : (FMT == BSQ_MXFP4) ? 16 : 8;
    static constexpr int kSfaCols = (FMT == BSQ_NVFP4) ? 16 : (FMT == BSQ_MXFP4) ? 8 : 4;
    static constexpr int kSfb0 = 256;
    static constexpr int kSfa0 = 256 + kStages * kSfbCols;
    static constexpr int kSfBoxRows = kSfaBytes / 256;  // SF tensor-map box height (rows of 256 B)
    static_assert(kSfa0 + kStages * kSfaCols <= 512, "TMEM budget");
    static_assert(kStages >= 2, "shared-memory budget");
};

template <int FMT, bool OUT_BF16, bool GROUPED, bool QOUT = false>
__global__ void __launch_bounds__(448, 1)
    gemm_bs2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                    const __grid_constant__ CUtensorMap tmC, const GemmParams p) {
    static_assert(!QOUT || OUT_BF16, "the quantizing epilogue quantizes the bf16 output");
    // the previous kernel in the stream has completed before anything here
    // (waiting after the set-up, as the single-CTA kernel does, measured slower)
    grid_dependency_wait();
    grid_dependents_launch();
    using C_ = Cfg2<FMT, GROUPED>;
    using T = typename C_::T;
    constexpr int NS = C_::kStages;
    constexpr int BN = 256;
    // One barrier wait per k-tile for the MMA thread (the leader's scale warps
    // fold the A/B arrival into sf_ready).  The quantizing epilogue keeps the
    // two separate waits: its kernel is bound by the epilogue warps, and there
    // the folded form measured slower (564 vs 520 us on the grouped up GEMM).
    constexpr bool kOneWait = !QOUT;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[NS], sf_full[NS], sf_ready[NS], empty_bar[NS], accf_bar, acce_bar,
        drain_bar;
    __shared__ uint32_t tmem_base_slot;
    __shared__ volatile int abort_flag;
    __shared__ int tile_start[GROUPED ? 1025 : 1];
    __shared__ int32_t offs[GROUPED ? 1025 : 1];
    __shared__ float q_den[QOUT ? 128 : 1], q_rcp[QOUT ? 128 : 1];

    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = sA + NS * C_::kABytes;
    uint8_t *sSFA = sB + NS * C_::kBBytes;
    uint8_t *sSFB = sSFA + NS * C_::kSfaBytes;
    uint8_t *sStage = smem + C_::kStagingOff;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int64_t m_tiles = (p.MA + 255) / 256;
    const int64_t n_tiles = (p.NB + BN - 1) / BN;
    const int64_t k_tiles = (p.K + T::kBkElems - 1) / T::kBkElems;
    const int64_t KBT = p.K / (T::kVec * 4);  // SF atoms per 128-row tile along K

    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; i++) {
            mbar_init(smem_u32(&full_bar[i]), 1);
            mbar_init(smem_u32(&sf_full[i]), 1);
            mbar_init(smem_u32(&sf_ready[i]), 2 * C_::kSfWarps);
            mbar_init(smem_u32(&empty_bar[i]), 1);
        }
        mbar_init(smem_u32(&accf_bar), 1);
        mbar_init(smem_u32(&acce_bar), 2 * C_::kEpiWarps);
        mbar_init(smem_u32(&drain_bar), 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        prefetch_tmap(&tmSFA);
        prefetch_tmap(&tmSFB);
        prefetch_tmap(&tmC);
    }
    int64_t total_tiles = m_tiles * n_tiles;
    if (GROUPED && warp == 2) {
        for (int i = lane; i <= p.G; i += 32) offs[i] = __ldg(p.row_off + i);
        __syncwarp();
        int carry = 0;
        for (int g0 = 0; g0 < p.G; g0 += 32) {
            int g = g0 + lane;
            int cnt = 0;
            if (g < p.G) cnt = ((offs[g + 1] - offs[g] + 255) / 256) * (int)n_tiles;
            int incl = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += v;
            }
            if (g < p.G) tile_start[g] = carry + incl - cnt;
            carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
        }
        if (lane == 0) tile_start[p.G] = carry;
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(&tmem_base_slot), 512);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // barriers of both CTAs are initialised before any remote arrive
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_slot;
    if (GROUPED) total_tiles = tile_start[p.G];

    // (group, 256-row m tile, n tile) of pair tile t; rows of this CTA
    auto info = [&](int64_t t, int64_t &a_row0, int64_t &sfa_row0, int64_t &m_lim, int64_t &nt, int &group) {
        if (!GROUPED) {
            const int64_t mt = t % m_tiles;
            nt = t / m_tiles;
            a_row0 = mt * 256 + 128 * rank;
            sfa_row0 = a_row0;
            m_lim = p.m_lim;
            group = 0;
            return;
        }
        int lo = 0, hi = p.G;
        while (hi - lo > 1) {
            int mid = (lo + hi) >> 1;
            if (tile_start[mid] <= t) lo = mid; else hi = mid;
        }
        const int64_t local = t - tile_start[lo];
        const int64_t mt_g = ((int64_t)offs[lo + 1] - offs[lo] + 255) / 256;
        const int64_t mt = local % mt_g;
        nt = local / mt_g;
        a_row0 = (int64_t)offs[lo] + mt * 256 + 128 * rank;
        sfa_row0 = (int64_t)__ldg(p.sf_row_off + lo) + mt * 256 + 128 * rank;
        m_lim = min((int64_t)offs[lo + 1], p.m_lim);
        group = lo;
    };

    // the leader's barriers, as seen from this CTA
    const uint32_t full0 = mapa(smem_u32(&full_bar[0]), 0);
    const uint32_t ready0 = mapa(smem_u32(&sf_ready[0]), 0);
    const uint32_t acce_leader = mapa(smem_u32(&acce_bar), 0);

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0, armed = 0, armed_par = 0;
            bool ok = true;
            constexpr uint32_t kPairBytes = 2 * (C_::kABytes + C_::kBBytes);
            constexpr uint32_t kSfBytes = C_::kSfaBytes + C_::kSfbBytes;
            for (int64_t t = pair; t < total_tiles && ok; t += npairs) {
                int64_t a_row0, sfa_row0, m_lim, nt;
                int group;
                info(t, a_row0, sfa_row0, m_lim, nt, group);
                const int64_t nb0 = nt * BN;
                const int64_t b_row0 = (int64_t)group * p.NB + nb0 + 128 * rank;
                // SF tensor maps address rows of 256 bytes
                const int64_t sfa_r0 = (sfa_row0 / 128) * KBT * 2;
                const int64_t sfb_r0 = (int64_t)group * (p.sfB_group_bytes / 256) + (nb0 / 128) * KBT * 2;
                for (int64_t kt = 0; kt < k_tiles; kt++) {
                    if (!mbar_wait(smem_u32(&empty_bar[s]), ph ^ 1u, &abort_flag, p.err, 1, kTimeoutNs)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = full0 + (uint32_t)(s * 8);  // leader's full barrier of stage s
                    if (leader) mbar_arrive_expect_tx(smem_u32(&full_bar[s]), kPairBytes);
                    const int32_t kx = (int32_t)(kt * 128);
                    tma_load_2d_pair(smem_u32(sA + s * C_::kABytes), &tmA, fb, kx, (int32_t)a_row0);
                    tma_load_2d_pair(smem_u32(sB + s * C_::kBBytes), &tmB, fb, kx, (int32_t)b_row0);
                    const uint32_t sb = smem_u32(&sf_full[s]);
                    const int32_t sfk = (int32_t)(kt * C_::kSfBoxRows);
                    mbar_arrive_expect_tx(sb, kSfBytes);
                    tma_load_2d(smem_u32(sSFA + s * C_::kSfaBytes), &tmSFA, sb, 0, (int32_t)(sfa_r0 + sfk));
                    tma_load_2d(smem_u32(sSFB + s * C_::kSfbBytes), &tmSFB, sb, 0, (int32_t)(sfb_r0 + sfk));
                    tma_load_2d(smem_u32(sSFB + s * C_::kSfbBytes + C_::kSfaBytes), &tmSFB, sb, 0,
                                (int32_t)(sfb_r0 + KBT * 2 + sfk));
                    armed |= 1u << s;
                    armed_par = (armed_par & ~(1u << s)) | (ph << s);
                    if (++s == NS) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            // before exit every copy this CTA started has landed: its own
            // scale tiles (sf_full), and -- through the leader's MMAs having
            // read them -- its A/B halves
            for (int i = 0; i < NS; i++)
                if (armed & (1u << i)) {
                    volatile int never = 0;
                    mbar_wait(smem_u32(&sf_full[i]), (armed_par >> i) & 1u, &never, p.err, 2, kTimeoutNs);
                    if (leader)
                        mbar_wait(smem_u32(&full_bar[i]), (armed_par >> i) & 1u, &never, p.err, 2, kTimeoutNs);
                    else if (!abort_flag)
                        mbar_wait(smem_u32(&empty_bar[i]), (armed_par >> i) & 1u, &abort_flag, p.err, 2, kTimeoutNs);
                }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader only)
        if (leader && lane == 0) {
            const uint32_t idesc = T::kIdescFmt | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
            constexpr uint32_t kOpHi = smem_desc_hi(1024, 2);  // K-major, 128-byte swizzle, 8-row groups 1 KB apart
            const uint32_t a_lo0 = smem_desc_lo(smem_u32(sA), 16), b_lo0 = smem_desc_lo(smem_u32(sB), 16);
            int s = 0;
            uint32_t ph = 0;
            bool ok = true, issued = false;
            int64_t it = 0;
            for (int64_t t = pair; t < total_tiles && ok; t += npairs, it++) {
                if (!mbar_wait(smem_u32(&acce_bar), (uint32_t)(it & 1) ^ 1u, &abort_flag, p.err, 3, kTimeoutNs)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int64_t kt = 0; kt < k_tiles; kt++) {
                    // kOneWait: sf_ready[s] completes after the stage's A/B
                    // halves have landed (the leader's scale warps wait for
                    // them) and both CTAs' scales are in TMEM, so it is the
                    // only wait per k-tile
                    if (!(kOneWait || mbar_test_wait(smem_u32(&full_bar[s]), ph) ||
                          mbar_wait(smem_u32(&full_bar[s]), ph, &abort_flag, p.err, 4, kTimeoutNs)) ||
                        !(mbar_test_wait(smem_u32(&sf_ready[s]), ph) ||
                          mbar_wait(smem_u32(&sf_ready[s]), ph, &abort_flag, p.err, 7, kTimeoutNs))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_lo = a_lo0 + (uint32_t)s * (C_::kABytes >> 4);
                    const uint32_t b_lo = b_lo0 + (uint32_t)s * (C_::kBBytes >> 4);
                    const uint32_t sfb_t = tmem_base + C_::kSfb0 + (uint32_t)s * C_::kSfbCols;
                    const uint32_t sfa_t = tmem_base + C_::kSfa0 + (uint32_t)s * C_::kSfaCols;
                    const int64_t krem = p.K - kt * T::kBkElems;
                    const int nmma = krem >= T::kBkElems ? C_::kMmaPerKt : (int)(krem / T::kMmaK);
                    auto one = [&](int j) {
                        const uint32_t acc = (kt > 0 || j > 0) ? 1u : 0u;
                        const uint64_t ad = desc_pack(a_lo + 2 * j, kOpHi), bd = desc_pack(b_lo + 2 * j, kOpHi);
                        if (FMT == BSQ_NVFP4) {
                            // MMA j: SFA at 4j (4-column aligned), SFB atoms at 8j and 8j + 4
                            mma_nvfp4_pair(tmem_base, ad, bd, idesc, sfa_t + 4 * j, sfb_t + 8 * j, acc);
                        } else if (FMT == BSQ_MXFP4) {
                            // MMA j: k-atom j / 2 (SFA at 4 (j / 2), SFB at 8 (j / 2)), scale
                            // bytes 2 (j % 2) and 2 (j % 2) + 1
                            const uint32_t id = 2u * (uint32_t)(j & 1), a = (uint32_t)(j >> 1);
                            mma_mxfp4_pair(tmem_base, ad, bd, idesc | (id << 29) | (id << 4), (sfa_t + 4 * a) | (id << 30),
                                           (sfb_t + 8 * a) | (id << 30), acc);
                        } else {
                            // scale byte j of each 32-bit column (scale-factor id)
                            mma_mxfp8_pair(tmem_base, ad, bd, idesc | ((uint32_t)j << 29) | ((uint32_t)j << 4),
                                           sfa_t | ((uint32_t)j << 30), sfb_t | ((uint32_t)j << 30), acc);
                        }
                    };
                    if (nmma == C_::kMmaPerKt) {
#pragma unroll
                        for (int j = 0; j < C_::kMmaPerKt; j++) one(j);
                    } else {
                        for (int j = 0; j < nmma; j++) one(j);
                    }
                    issued = true;
                    tc_commit_pair(smem_u32(&empty_bar[s]), 0x3);  // release stage s in both CTAs
                    if (++s == NS) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit_pair(smem_u32(&accf_bar), 0x3);
            }
            if (issued) {
                tc_commit_pair(smem_u32(&drain_bar), 0x1);
                volatile int never = 0;
                mbar_wait(smem_u32(&drain_bar), 0, &never, p.err, 5, kTimeoutNs);
            }
        }
    } else if (warp < 2 + C_::kSfWarps) {
        // ------------------------------------------------------------ scale warps (both CTAs)
        const int q = warp & 3;  // the TMEM lane quarter this warp may write
        const uint32_t lane_base = tmem_base + ((uint32_t)(32 * q) << 16);
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int64_t t = pair; t < total_tiles && ok; t += npairs) {
            for (int64_t kt = 0; kt < k_tiles; kt++) {
                // warp-uniform decisions: tcgen05.st is warp-collective
                ok = __all_sync(0xFFFFFFFFu,
                                mbar_wait(smem_u32(&sf_full[s]), ph, &abort_flag, p.err, 8, kTimeoutNs));
                if (!ok) break;
                const uint8_t *sfa = sSFA + s * C_::kSfaBytes;
                const uint8_t *sfb = sSFB + s * C_::kSfbBytes;
                const uint32_t sfb_t = lane_base + C_::kSfb0 + (uint32_t)s * C_::kSfbCols;
                const uint32_t sfa_t = lane_base + C_::kSfa0 + (uint32_t)s * C_::kSfaCols;
                // an atom holds rows r, r+32, r+64, r+96 of its 128 in the 16 bytes at 16 (r % 32)
                if (FMT == BSQ_NVFP4) {
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        // SFB of MMA j: both 128-row atoms, replicated in every quarter
                        const uint4 b0 = *reinterpret_cast<const uint4 *>(sfb + 512 * j + 16 * lane);
                        const uint4 b1 = *reinterpret_cast<const uint4 *>(sfb + C_::kSfaBytes + 512 * j + 16 * lane);
                        const uint32_t w[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                        tmem_st_x8(sfb_t + 8 * j, w);
                        // SFA of MMA j: this quarter's rows, in the column the quarter reads
                        tmem_st_x1(sfa_t + 4 * j + q, *reinterpret_cast<const uint32_t *>(sfa + 512 * j + 16 * lane + 4 * q));
                    }
                } else if (FMT == BSQ_MXFP4) {
#pragma unroll
                    for (int a = 0; a < 2; a++) {
                        // k-atom a: SFB of both 128-row atoms (every quarter), SFA of this quarter
                        const uint4 b0 = *reinterpret_cast<const uint4 *>(sfb + 512 * a + 16 * lane);
                        const uint4 b1 = *reinterpret_cast<const uint4 *>(sfb + C_::kSfaBytes + 512 * a + 16 * lane);
                        const uint32_t w[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                        tmem_st_x8(sfb_t + 8 * a, w);
                        tmem_st_x1(sfa_t + 4 * a + q,
                                   *reinterpret_cast<const uint32_t *>(sfa + 512 * a + 16 * lane + 4 * q));
                    }
                } else {
                    const uint4 b0 = *reinterpret_cast<const uint4 *>(sfb + 16 * lane);
                    const uint4 b1 = *reinterpret_cast<const uint4 *>(sfb + C_::kSfaBytes + 16 * lane);
                    const uint32_t w[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                    tmem_st_x8(sfb_t, w);
                    tmem_st_x1(sfa_t + q, *reinterpret_cast<const uint32_t *>(sfa + 16 * lane + 4 * q));
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (kOneWait && leader) {
                    // the leader's warps also wait for the stage's A/B halves
                    // (both CTAs' copies complete on the leader's full_bar) and
                    // pass them on with a CTA-scope release arrive
                    bool landed = true;
                    if (lane == 0) landed = mbar_wait(smem_u32(&full_bar[s]), ph, &abort_flag, p.err, 4, kTimeoutNs);
                    ok = __shfl_sync(0xFFFFFFFFu, landed, 0);
                    if (!ok) break;
                    if (lane == 0) mbar_arrive(smem_u32(&sf_ready[s]));
                } else if (lane == 0) {
                    mbar_arrive_cluster_relaxed(ready0 + (uint32_t)(s * 8));
                }
                if (++s == NS) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int ew = warp - 2 - C_::kSfWarps;  // 0..7
        const int q = warp & 3;
        const int half = ew >> 2;
        constexpr int HC = BN / 2;
        uint8_t *box_base = sStage + ew * C_::kBoxes * C_::kBoxBytes;
        // 64-byte swizzle of a 32-row x 64-byte box: 16-byte chunk c of row r
        // sits at chunk c ^ ((r >> 1) & 3) (the pattern the tensor map names)
        auto box_addr = [&](int box, int c) -> uint8_t * {
            return box_base + box * C_::kBoxBytes + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4);
        };
        auto put_row = [&](int box, const uint32_t (&v)[16]) {
#pragma unroll
            for (int c = 0; c < 4; c++)
                *reinterpret_cast<uint4 *>(box_addr(box, c)) = make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
        };
        auto get_row = [&](int box, uint32_t (&v)[16]) {
#pragma unroll
            for (int c = 0; c < 4; c++) {
                const uint4 w = *reinterpret_cast<const uint4 *>(box_addr(box, c));
                v[4 * c] = w.x;
                v[4 * c + 1] = w.y;
                v[4 * c + 2] = w.z;
                v[4 * c + 3] = w.w;
            }
        };
        // quantizing epilogue: the NVFP4 tables of the given global scale
        // (den / rcp per E4M3 code), built by the 256 epilogue threads
        NvScale qs{};
        if (QOUT) {
            const float s_g = __ldg(p.q_sg);
            const int et = ew * 32 + lane;
            if (et < 128) {
                const float den = __fmul_rn(e4m3_to_f32(et), s_g);
                q_den[et] = den;
                q_rcp[et] = (et == 0 || et == 127) ? 0.0f : __frcp_rn(den);
            }
            asm volatile("bar.sync 2, %0;" ::"n"(32 * C_::kEpiWarps) : "memory");
            qs.s_g = s_g;
            qs.c6 = __frcp_rn(__fmul_rn(6.0f, s_g));
            qs.c4 = __frcp_rn(__fmul_rn(4.0f, s_g));
            qs.fast = s_g >= 0x1p-90f && s_g <= 0x1p100f;
        }
        int64_t it = 0;
        int nstored = 0;  // boxes this warp has handed to TMA (fp32 path: ring position)
        for (int64_t t = pair; t < total_tiles; t += npairs, it++) {
            int64_t a_row0, sfa_row0, m_lim, nt;
            int group;
            info(t, a_row0, sfa_row0, m_lim, nt, group);
            float alpha = 1.0f;  // read before the wait: off the drain's critical path
            if (FMT == BSQ_NVFP4) {
                const float ga = p.gsA ? __ldg(p.gsA) : 1.0f;
                const float gb = p.gsB ? __ldg(p.gsB + group) : 1.0f;
                alpha = __fmul_rn(ga, gb);
            }
            if (!mbar_wait(smem_u32(&accf_bar), (uint32_t)(it & 1), &abort_flag, p.err, 6, kTimeoutNs)) break;
            tc_fence_after();
            const int64_t row0 = a_row0 + 32 * q;  // first row of this warp's boxes
            const int64_t ar = row0 + lane;
            const bool row_ok = ar < m_lim;
            const bool box_rows_ok = row0 + 32 <= m_lim;  // TMA boxes never cross a group's end
            const int64_t nb0 = nt * BN + half * HC;
            const int64_t n_lim = p.n_lim;
            const uint32_t tbase = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(half * HC);
            if (OUT_BF16) {
                // drain this warp's 128 columns into registers (bf16-packed) and
                // release the accumulator before any store
                uint32_t pk[HC / 2];
#pragma unroll
                for (int c = 0; c < HC / 32; c += 2) {
                    // two 32-column loads in flight per wait
                    uint32_t r0[32], r1[32];
                    tmem_ld32(tbase + 32 * c, r0);
                    tmem_ld32(tbase + 32 * c + 32, r1);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 16; j++) {
                        __nv_bfloat162 h = __floats2bfloat162_rn(__fmul_rn(alpha, __uint_as_float(r0[2 * j])),
                                                                 __fmul_rn(alpha, __uint_as_float(r0[2 * j + 1])));
                        pk[16 * c + j] = *reinterpret_cast<uint32_t *>(&h);
                    }
#pragma unroll
                    for (int j = 0; j < 16; j++) {
                        __nv_bfloat162 h = __floats2bfloat162_rn(__fmul_rn(alpha, __uint_as_float(r1[2 * j])),
                                                                 __fmul_rn(alpha, __uint_as_float(r1[2 * j + 1])));
                        pk[16 * c + 16 + j] = *reinterpret_cast<uint32_t *>(&h);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster_relaxed(acce_leader);
                if (QOUT) {
                    // NVFP4 of this thread's 128 bf16 outputs (eight blocks of 16,
                    // block b = pk[8b .. 8b + 7]), quantized as bsq_quant_nvfp4
                    // does with the given global scale; codes and swizzled scale
                    // words stored directly; max |output| kept for the next scale
                    uint32_t amax_bits = 0u;
                    if (row_ok) {
                        const int64_t sf_row = sfa_row0 + 32 * q + lane;
                        const int64_t qkb = p.NB >> 4;
                        const uint32_t sw0[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
                        for (int g4 = 0; g4 < 2; g4++) {
                            const int64_t n4 = nb0 + 64 * g4;   // first column of 4 blocks
                            if (n4 >= n_lim) break;
                            uint32_t sbw = 0u;
                            uint2 cd[4];
#pragma unroll
                            for (int i = 0; i < 4; i++) {
                                const uint32_t *w = pk + 8 * (4 * g4 + i);
                                uint32_t sb;
                                if (p.q_fos) nv_block_1d<false, true>(w, sw0, qs, q_den, q_rcp, sb, cd[i]);
                                else nv_block_1d<false, false>(w, sw0, qs, q_den, q_rcp, sb, cd[i]);
                                sbw |= (sb & 0xFFu) << (8 * i);
#pragma unroll
                                for (int k = 0; k < 8; k++) amax_bits = max(amax_bits, max(w[k] & 0x7FFFu, (w[k] >> 16) & 0x7FFFu));
                            }
                            uint4 *cp = reinterpret_cast<uint4 *>(p.q_codes + ar * (p.NB >> 1) + (n4 >> 1));
                            cp[0] = make_uint4(cd[0].x, cd[0].y, cd[1].x, cd[1].y);
                            cp[1] = make_uint4(cd[2].x, cd[2].y, cd[3].x, cd[3].y);
                            *reinterpret_cast<uint32_t *>(p.q_sf + sf_word_offset(sf_row, n4 >> 6, qkb)) = sbw;
                        }
                    }
                    if (p.q_amax) {
#pragma unroll
                        for (int o = 16; o; o >>= 1) amax_bits = max(amax_bits, __shfl_xor_sync(0xFFFFFFFFu, amax_bits, o));
                        // bf16 magnitude bits << 16 are the fp32 bits of the same value
                        if (lane == 0 && amax_bits) atomicMax(p.q_amax, amax_bits << 16);
                    }
                    if (p.C == nullptr) continue;
                }
#pragma unroll
                for (int c = 0; c < HC / 32; c++) {
                    const int64_t n = nb0 + 32 * c;
                    uint32_t v[16];
#pragma unroll
                    for (int j = 0; j < 16; j++) v[j] = pk[16 * c + j];
                    if (n >= n_lim) {
                        // past the last column: nothing to store
                    } else if (box_rows_ok) {
                        const int box = nstored & (C_::kBoxes - 1);
                        if (nstored >= C_::kBoxes) {
                            if (lane == 0) bulk_wait_read<C_::kBoxes - 1>();  // this box's last store has read it
                            __syncwarp();
                        }
                        put_row(box, v);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tmC, smem_u32(box_base + box * C_::kBoxBytes), (int32_t)n, (int32_t)row0);
                            bulk_commit();
                        }
                        nstored++;
                    } else if (row_ok) {
                        uint16_t *dst = reinterpret_cast<uint16_t *>(static_cast<__nv_bfloat16 *>(p.C) + ar * p.ldc + n);
                        for (int j = 0; j < 32; j++)
                            if (n + j < n_lim) dst[j] = (j & 1) ? (uint16_t)(v[j / 2] >> 16) : (uint16_t)(v[j / 2] & 0xFFFFu);
                    }
                }
            } else {
                // fp32: 16-column boxes through the box ring; the accumulator is
                // released after the last load
#pragma unroll 1
                for (int c = 0; c < HC / 16; c++) {
                    uint32_t r[16];
                    tmem_ld16(tbase + 16 * c, r);
                    tmem_ld_wait();
                    if (c == HC / 16 - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster_relaxed(acce_leader);
                    }
                    const int64_t n = nb0 + 16 * c;
                    if (n >= n_lim) continue;
                    uint32_t v[16];
#pragma unroll
                    for (int j = 0; j < 16; j++) v[j] = __float_as_uint(__fmul_rn(alpha, __uint_as_float(r[j])));
                    if (box_rows_ok) {
                        const int box = nstored & (C_::kBoxes - 1);
                        if (nstored >= C_::kBoxes) {
                            if (lane == 0) bulk_wait_read<C_::kBoxes - 1>();  // this box's last store has read it
                            __syncwarp();
                        }
                        put_row(box, v);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tmC, smem_u32(box_base + box * C_::kBoxBytes), (int32_t)n, (int32_t)row0);
                            bulk_commit();
                        }
                        nstored++;
                    } else if (row_ok) {
                        float *dst = static_cast<float *>(p.C) + ar * p.ldc + n;
                        for (int j = 0; j < 16; j++)
                            if (n + j < n_lim) dst[j] = __uint_as_float(v[j]);
                    }
                }
            }
        }
        // every store of this warp has completed before the CTA exits
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the peer's shared memory stays valid until the pair is done
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, 512);
    }
}

// ============================================================ timeout probe
__global__ void timeout_probe_kernel(uint64_t timeout_ns, unsigned int *err) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ volatile int abort_flag;
    if (threadIdx.x == 0) {
        sm100::mbar_init(sm100::smem_u32(&bar), 1);
        abort_flag = 0;
        sm100::fence_barrier_init();
        // nobody arrives: the wait must run out and report site 15
        sm100::mbar_wait(sm100::smem_u32(&bar), 0, &abort_flag, err, 15, timeout_ns);
    }
}

void launch_timeout_probe(uint64_t timeout_ns, unsigned int *err, cudaStream_t s) {
    timeout_probe_kernel<<<1, 32, 0, s>>>(timeout_ns, err);
}

// ============================================================ host side
// The dynamic shared-memory limit of a kernel is a per-device attribute:
// set it once per (kernel, device), under a lock; a success is remembered.
int smem_attr_once(const void *kern, int bytes) {
    static PerDeviceMemo<1024> done;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return BSQ_ERR_CUDA;
    return done.get(
        kern, dev,
        [&] {
            return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess
                       ? BSQ_OK
                       : BSQ_ERR_CUDA;
        },
        [](int st) { return st == BSQ_OK; });
}

namespace {

using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                              const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn get_encode() {
    static EncodeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeFn>(ptr);
    });
    return fn;
}

// 2-D uint8 tensor map: rows x row_bytes, box 128 bytes x box_rows, 128-byte swizzle.
bool make_tmap(CUtensorMap *m, const void *base, int64_t row_bytes, int64_t rows, int box_rows) {
    EncodeFn enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


// 2-D uint8 tensor map over a scale-factor buffer seen as rows of 256 bytes.
bool make_sf_tmap(CUtensorMap *m, const void *base, int64_t bytes, int box_rows) {
    EncodeFn enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {256u, (cuuint64_t)(bytes / 256)};
    cuuint64_t strides[1] = {256u};
    cuuint32_t box[2] = {256u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D tensor map over the output C (rows x n_cols elements, row stride ldc):
// 32-row boxes of 64 bytes (32 bf16 or 16 fp32 columns), 64-byte swizzle,
// for the pair kernel's TMA-store epilogue.
bool make_c_tmap(CUtensorMap *m, void *C, bool bf16, int64_t n_cols, int64_t rows, int64_t ldc) {
    EncodeFn enc = get_encode();
    if (!enc) return false;
    const int64_t esz = bf16 ? 2 : 4;
    cuuint64_t dims[2] = {(cuuint64_t)n_cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(ldc * esz)};
    cuuint32_t box[2] = {(cuuint32_t)(64 / esz), 32u};
    cuuint32_t estr[2] = {1u, 1u};
    return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, C, dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 C [rows][ld] seen as (n_cols x rows) tiles of box_cols x box_rows,
// no swizzle (the staging tile is plain row-major)
bool make_c_tmap_box(CUtensorMap *m, void *C, int64_t n_cols, int64_t rows, int64_t ldc, int box_cols, int box_rows) {
    EncodeFn enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)n_cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(ldc * 2)};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, C, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

template <int FMT, bool OUT_BF16, bool GROUPED, bool QOUT = false>
int run_pair(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tsa, const CUtensorMap &tsb,
             const CUtensorMap &tc, const GemmParams &p, int pairs, cudaStream_t s) {
    using C_ = Cfg2<FMT, GROUPED>;
    auto kern = gemm_bs2_kernel<FMT, OUT_BF16, GROUPED, QOUT>;
    if (smem_attr_once(reinterpret_cast<const void *>(kern), C_::kSmemBytes) != BSQ_OK) return BSQ_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    cfg.blockDim = dim3(C_::kThreads, 1, 1);
    cfg.dynamicSmemBytes = C_::kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // the kernel waits for the previous one (grid_dependency_wait) before any global access
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = kernel_choice(BSQ_KNOB_LAUNCH_OVERLAP) != 0 ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, kern, ta, tb, tsa, tsb, tc, p) != cudaSuccess) return BSQ_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? BSQ_OK : BSQ_ERR_CUDA;
}

template <int FMT, int BN, int ACC, bool OUT_BF16, bool SWAP, bool GROUPED>
int run(const CUtensorMap &ta, const CUtensorMap &tb, const GemmParams &p, int grid, cudaStream_t s,
        const CUtensorMap *tc = nullptr) {
    using C_ = Cfg<FMT, BN>;
    auto kern = gemm_bs_kernel<FMT, BN, ACC, OUT_BF16, SWAP, GROUPED>;
    if (smem_attr_once(reinterpret_cast<const void *>(kern), C_::kSmemBytes) != BSQ_OK) return BSQ_ERR_CUDA;
    if (launch_dependent(kern, grid, C_::kThreads, C_::kSmemBytes, s, ta, tb, tc ? *tc : ta, p) != cudaSuccess)
        return BSQ_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? BSQ_OK : BSQ_ERR_CUDA;
}

// The swap-AB kernel split over K: clusters of S CTAs, one tile per cluster.
template <int FMT, bool OUT_BF16, int S>
int run_splitk(const CUtensorMap &ta, const CUtensorMap &tb, const GemmParams &p, int64_t tiles, cudaStream_t s) {
    using C_ = Cfg<FMT, 64, 3>;
    auto kern = gemm_bs_kernel<FMT, 64, 2, OUT_BF16, true, false, S>;
    if (smem_attr_once(reinterpret_cast<const void *>(kern), C_::kSmemBytes) != BSQ_OK) return BSQ_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(tiles * S), 1, 1);
    cfg.blockDim = dim3(C_::kThreads, 1, 1);
    cfg.dynamicSmemBytes = C_::kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = S;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // the kernel waits for the previous one (grid_dependency_wait) before any global access
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = kernel_choice(BSQ_KNOB_LAUNCH_OVERLAP) != 0 ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, kern, ta, tb, ta, p) != cudaSuccess) return BSQ_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? BSQ_OK : BSQ_ERR_CUDA;
}

template <int FMT>
int dispatch(const GemmArgs &g, cudaStream_t s) {
    using T = FmtTraits<FMT>;
    const int64_t kb_bytes = (FMT == BSQ_MXFP8) ? g.K : g.K / 2;
    const bool grouped = g.G > 0;
    const bool swap = !grouped && g.M <= 64 && g.N >= 128;
    // operand A supplies the 128-row MMA dimension
    const uint8_t *opA = swap ? g.B : g.A, *opB = swap ? g.A : g.B;
    const uint8_t *sfA = swap ? g.sfB : g.sfA, *sfB = swap ? g.sfA : g.sfB;
    const float *gsA = swap ? g.gsB : g.gsA, *gsB = swap ? g.gsA : g.gsB;
    const int64_t MA = swap ? g.N : g.M, NB = swap ? g.M : g.N;
    int bn;
    if (swap) bn = 64;
    else if (g.out_bf16 && NB >= 256) bn = 256;
    else bn = 128;
    // CTA pairs (256x256 tiles) for large operands: on 8192x14336x4096 NVFP4
    // they measure 4.50 PFLOP/s against 3.24 for single-CTA 128x256 tiles.
    // Single CTAs keep the skinny swap-AB case, operands with fewer than 256
    // rows, outputs that TMA cannot store (unaligned base or row stride) and
    // grouped NVFP4 with a half k-tile (that would need the exact extent of
    // A's scale buffer, which only the device knows).  The BSQ_KNOB_GEMM_PAIR
    // override forces either kernel where the pair kernel is possible
    // (tuning, tests).
    const int64_t c_esz = g.out_bf16 ? 2 : 4;
    const bool qout = g.q_codes != nullptr;
    const bool c_tma_ok = (g.C == nullptr && qout) ||
                          ((reinterpret_cast<uintptr_t>(g.C) % 16 == 0) && (g.ldc * c_esz) % 16 == 0);
    const bool pair_ok = !swap && NB >= 128 && c_tma_ok && !(FMT != BSQ_MXFP8 && g.K % 256 != 0);
    bool use_pair = pair_ok && MA >= 256 && NB >= 256;
    if (const int v = kernel_choice(BSQ_KNOB_GEMM_PAIR); v >= 0) use_pair = pair_ok && v != 0;
    if (qout) {
        // the quantizing epilogue exists in the pair kernel only
        if (!pair_ok || !grouped || !g.out_bf16 || FMT != BSQ_NVFP4) return BSQ_ERR_UNSUPPORTED;
        use_pair = true;
    }
    if (const int v = kernel_choice(BSQ_KNOB_GEMM_BN); v > 0) {  // tuning override of the single-CTA tile
        if ((v == 128 || (v == 256 && g.out_bf16)) && !swap) bn = v;
    }
    GemmParams p{};
    p.sfA = sfA; p.sfB = sfB; p.gsA = gsA; p.gsB = gsB;
    p.MA = MA; p.NB = NB; p.K = g.K;
    p.m_lim = MA; p.n_lim = NB;
    p.C = g.C; p.ldc = g.ldc;
    p.sfB_group_bytes = (int64_t)((NB + 127) / 128 * 128) * ((g.K / T::kVec + 3) / 4 * 4);
    p.G = g.G; p.row_off = g.row_off; p.sf_row_off = g.sf_row_off;
    p.err = g.err;
    p.q_codes = g.q_codes; p.q_sf = g.q_sf; p.q_sg = g.q_sg; p.q_amax = g.q_amax; p.q_fos = g.q_fos ? 1 : 0;
    CUtensorMap ta, tb;
    if (!make_tmap(&ta, opA, kb_bytes, MA, 128)) return BSQ_ERR_CUDA;
    if (use_pair) {
        CUtensorMap tsa, tsb;
        if (!make_tmap(&tb, opB, kb_bytes, grouped ? (int64_t)g.G * NB : NB, 128)) return BSQ_ERR_CUDA;
        const int64_t kbp = (g.K / T::kVec + 3) / 4 * 4;
        const int64_t sfa_rows = grouped ? 0 : (MA + 127) / 128 * 128;
        // grouped A: the SF buffer spans sf_row_offsets[G] rows; its size is not
        // known on the host, so map the largest extent the groups can reach
        const int64_t sfa_bytes = grouped ? ((MA + 128LL * g.G + 127) / 128 * 128) * kbp : sfa_rows * kbp;
        const int64_t sfb_bytes = (grouped ? (int64_t)g.G : 1) * p.sfB_group_bytes;
        const int box = Cfg2<FMT, false>::kSfBoxRows;
        if (!make_sf_tmap(&tsa, sfA, sfa_bytes, box) || !make_sf_tmap(&tsb, sfB, sfb_bytes, box)) return BSQ_ERR_CUDA;
        CUtensorMap tc;
        // without a bf16 output the store map is never used: give it the code
        // buffer's own extent (rows of NB/2 bytes seen as NB/4 bf16)
        if (g.C == nullptr ? !make_c_tmap(&tc, g.q_codes, true, NB / 4, MA, NB / 4)
                           : !make_c_tmap(&tc, g.C, g.out_bf16, NB, MA, g.ldc))
            return BSQ_ERR_CUDA;
        int64_t ptiles = grouped ? (MA / 256 + g.G) * ((NB + 255) / 256) : ((MA + 255) / 256) * ((NB + 255) / 256);
        int pairs = (int)(ptiles < g.num_sms / 2 ? (ptiles < 1 ? 1 : ptiles) : g.num_sms / 2);
        if (grouped) {
            if constexpr (FMT == BSQ_NVFP4) {
                if (qout) return run_pair<FMT, true, true, true>(ta, tb, tsa, tsb, tc, p, pairs, s);
            }
            if (g.out_bf16) return run_pair<FMT, true, true>(ta, tb, tsa, tsb, tc, p, pairs, s);
            return run_pair<FMT, false, true>(ta, tb, tsa, tsb, tc, p, pairs, s);
        }
        if (g.out_bf16) return run_pair<FMT, true, false>(ta, tb, tsa, tsb, tc, p, pairs, s);
        return run_pair<FMT, false, false>(ta, tb, tsa, tsb, tc, p, pairs, s);
    }
    if (!make_tmap(&tb, opB, kb_bytes, grouped ? (int64_t)g.G * NB : NB, bn)) return BSQ_ERR_CUDA;
    int64_t tiles;
    if (!grouped) tiles = ((MA + 127) / 128) * ((NB + bn - 1) / bn);
    else tiles = (MA / 128 + g.G) * ((NB + bn - 1) / bn);
    const int grid = (int)(tiles < g.num_sms ? (tiles < 1 ? 1 : tiles) : g.num_sms);
    if (swap) {
        // Split K when the tiles leave SMs idle: two split-K CTAs share an SM
        // (3 stages, 256 TMEM columns each), so S = 2, 4 or 8 is taken as
        // long as tiles x S fits twice the SM count and every CTA keeps at
        // least two k-tiles.  Not for NVFP4, whose unsplit kernel has the
        // scale-copier threads: on 64x14336x4096 it measures 15.9 us against
        // 16.7 split in two (MXFP4: 18.3 unsplit, 16.0 split).
        // BSQ_KNOB_GEMM_SPLITK forces S (1: off).
        const int64_t k_tiles = (g.K + T::kBkElems - 1) / T::kBkElems;
        int S = 1;
        while (FMT != BSQ_NVFP4 && S < 8 && tiles * (2 * S) <= 2LL * g.num_sms && k_tiles >= 2 * (2 * S)) S *= 2;
        if (const int v = kernel_choice(BSQ_KNOB_GEMM_SPLITK); v > 0) S = v;
        while (S > 1 && S > k_tiles) S /= 2;
        if (S == 2) return g.out_bf16 ? run_splitk<FMT, true, 2>(ta, tb, p, tiles, s) : run_splitk<FMT, false, 2>(ta, tb, p, tiles, s);
        if (S == 4) return g.out_bf16 ? run_splitk<FMT, true, 4>(ta, tb, p, tiles, s) : run_splitk<FMT, false, 4>(ta, tb, p, tiles, s);
        if (S == 8) return g.out_bf16 ? run_splitk<FMT, true, 8>(ta, tb, p, tiles, s) : run_splitk<FMT, false, 8>(ta, tb, p, tiles, s);
        if (g.out_bf16) {
            // the bf16 tile goes out as one TMA store ([tokens][W rows] of C)
            // when C's base and row stride suit TMA
            CUtensorMap tc;
            if ((reinterpret_cast<uintptr_t>(g.C) % 16) == 0 && (g.ldc * 2) % 16 == 0 &&
                make_c_tmap_box(&tc, g.C, MA, NB, g.ldc, 128, 64)) {
                p.c_tma = 1;
                return run<FMT, 64, 2, true, true, false>(ta, tb, p, grid, s, &tc);
            }
            return run<FMT, 64, 2, true, true, false>(ta, tb, p, grid, s);
        }
        return run<FMT, 64, 2, false, true, false>(ta, tb, p, grid, s);
    }
    if (grouped) {
        if (bn == 256) return run<FMT, 256, 1, true, false, true>(ta, tb, p, grid, s);
        if (g.out_bf16) return run<FMT, 128, 2, true, false, true>(ta, tb, p, grid, s);
        return run<FMT, 128, 2, false, false, true>(ta, tb, p, grid, s);
    }
    if (bn == 256) return run<FMT, 256, 1, true, false, false>(ta, tb, p, grid, s);
    if (g.out_bf16) return run<FMT, 128, 2, true, false, false>(ta, tb, p, grid, s);
    return run<FMT, 128, 2, false, false, false>(ta, tb, p, grid, s);
}

}  // namespace

int launch_gemm(const GemmArgs &g, cudaStream_t s) {
    if (g.fmt == BSQ_NVFP4) return dispatch<BSQ_NVFP4>(g, s);
    if (g.fmt == BSQ_MXFP4) return dispatch<BSQ_MXFP4>(g, s);
    return dispatch<BSQ_MXFP8>(g, s);
}

}  // namespace bsq
