// Block-scaled MXFP8 GEMM for sm_100a:
//
//   C[i][j] = sum_k (a_ik 2^(sfa[i][k/32]-127)) (b_kj 2^(sfb[j][k/32]-127))
//
// with FP8 E4M3 A (M x K) and K-major B (N x K), one E8M0 scale per 32
// consecutive K elements of every row, fp32 accumulation in TMEM and bf16 C.
// This is the block-scaled MMA of "Modern GPU Programming For MLSys - 书籍总结"
// (omica.com.cn), sections 2.4 and 2.6: the scale factors live in tensor
// memory and the tensor core applies them inside the MMA.
//
// Two kernels:
//   mxf8_repack_scales_kernel  turns the row-major scale bytes into 512-byte
//       chunks, one per (128-row block, 128-wide K block), laid out the way
//       tcgen05.cp 32x128b.warpx4 places them in TMEM: chunk byte
//       r*16 + q*4 + j holds the scale of row 32q + r for the j-th 32-wide
//       K step.  Padding rows and K steps get 127 (2^0), so zero-filled
//       operand tails stay zero.
//   (The GEMM is launched as a programmatic dependent of the repack: the
//   repack lets it start at once, and its producer waits for the repack grid
//   before the first load, so the GEMM's prologue overlaps the repack.)
//   gemm_mxf8_sm100_kernel  persistent, warp-specialised, one CTA (CG = 1,
//       128 x 256 tile) or a CTA pair (CG = 2, 256 x 256 tile, cta_group::2)
//       per tile, BK = 128 (one 128-byte swizzle row of E4M3):
//       warp 0 loads A, B and the scale chunks by TMA (for a pair, every
//       byte counts on the leader's barrier; each CTA holds its own 128 rows
//       of A scales and the scales of all 256 rows of B);
//       warp 10 of the (leader) CTA copies each stage's scales into one of
//       four TMEM scale slots (tcgen05.cp, cta_group::2 for a pair: each
//       CTA's SMEM to its own TMEM), ordered against the MMAs only by the
//       sf_full / sf_empty barriers, so a later stage's copy can overlap the
//       current stage's MMAs;
//       warp 1 of the (leader) CTA issues 4 block-scaled MMAs per stage
//       (K = 32 each, the byte of the scale column chosen in the instruction
//       descriptor);
//       warps 2-9 (two per TMEM lane quarter, half of the columns each)
//       drain the single-buffered accumulator into registers as packed
//       bf16, release TMEM, and only then write C with 16-byte global
//       stores, so the next tile's MMAs wait for the TMEM reads alone.
//
// TMEM: accumulator columns [0, 256); scale slot s at 256 + 32 s (A: 4
// columns) and 256 + 32 s + 16 (B: 8 columns).  Every scale sits in lane
// (row % 32) of each 32-lane quarter, column (row / 32), byte j.
#pragma once
#include <cstdint>

#include "gemm_bf16_sm100.cuh"
#include "ptx.cuh"

namespace b200 {

// Watchdog codes of the scale copier (role) and the scale-slot barriers.
constexpr int kRoleSfCopy = 5;
constexpr int kBarSfFull = 8, kBarSfEmpty = 9;

template <int CG_, int STAGES_>
struct GemmMxf8Cfg {
    static constexpr int CG = CG_;                 // CTAs per tile (cta_group)
    static constexpr int STAGES = STAGES_;
    static constexpr int BM_CTA = 128;             // accumulator rows per CTA
    static constexpr int BM = 128 * CG;            // tile M == MMA M
    static constexpr int BN = 256;                 // tile N == MMA N
    static constexpr int B_ROWS = BN / CG;         // rows of B this CTA loads
    static constexpr int BK = 128;                 // E4M3 elements (bytes) per k-tile
    static constexpr int UMMA_K = 32;              // K per block-scaled MMA
    static constexpr int MMAS = BK / UMMA_K;       // 4, one scale byte each
    static constexpr int A_BYTES = BM_CTA * BK;
    static constexpr int B_BYTES = B_ROWS * BK;
    static constexpr int SF_CHUNK = 512;           // scales of 128 rows x 4 K steps
    static constexpr int SFA_BYTES = SF_CHUNK;     // this CTA's 128 rows of A
    static constexpr int SFB_BYTES = 2 * SF_CHUNK; // all 256 rows of B (every CTA needs them)
    static constexpr int CTA_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr int TX_BYTES = CTA_BYTES * CG;  // bytes landing on the leader's full[s]
    static constexpr int STAGE_BYTES = ((CTA_BYTES + 1023) / 1024) * 1024;
    static constexpr int EPI_COLS = BN / 2;        // accumulator columns one epilogue warp drains
    static_assert(EPI_COLS % 64 == 0, "the drain reads 64 columns per TMEM round trip");
    // Scale slots in TMEM (32 columns each, beside the accumulator): a
    // separate warp copies stage s's scales into slot s % SF_SLOTS ahead of
    // the MMAs that read them.
    static constexpr int SF_SLOTS = 4;
    // full[S], empty[S], tmem_full, tmem_empty, sf_full[SF_SLOTS], sf_empty[SF_SLOTS]
    static constexpr int NUM_BARS = 2 * STAGES + 2 + 2 * SF_SLOTS;
    static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
    static constexpr int SMEM_BYTES = 1024 + BAR_OFF + NUM_BARS * 8 + 16;
    static constexpr int TMEM_COLS = 512;
    static constexpr int SF_COL0 = 256;
    // warp 0 producer, warp 1 MMA, warps 2-9 epilogue (two per TMEM lane
    // quarter, each draining half of the columns), warp 10 scale copier
    static constexpr int EPI_WARPS = 8;
    static constexpr int THREADS = 32 * (3 + EPI_WARPS);
    static_assert(SF_COL0 + 32 * SF_SLOTS <= TMEM_COLS, "scale slots fit beside the accumulator");
    static_assert(CG == 1 || CG == 2, "cta_group is 1 or 2");
    static_assert(B_ROWS % 8 == 0 && B_ROWS <= 256, "TMA box rows");
    static_assert(SMEM_BYTES <= 232448, "dynamic shared memory per CTA on sm_100");
};

// Row-major scales [rows][K/32] -> chunks [row block][K block][512], for
// a_blocks row blocks of A followed by b_blocks row blocks of B; rows past
// M (or N) and K steps past k32 read as 127.
//
// One CTA (256 threads) per (row block, group of kRepackKb K blocks): it
// reads the 128 rows x (4 kRepackKb) scale bytes coalesced into shared
// memory, then writes kRepackKb consecutive 512-byte chunks with 16-byte
// stores (thread r of a chunk writes the four words of rows r, r+32, r+64,
// r+96).
constexpr int kRepackKb = 8;

__global__ void __launch_bounds__(256)
mxf8_repack_scales_kernel(const uint8_t *__restrict__ sfa, int64_t M, int64_t a_blocks,
                          const uint8_t *__restrict__ sfb, int64_t N, int64_t b_blocks,
                          int64_t k32, int64_t kblocks, uint32_t *__restrict__ out) {
    // the GEMM launched after this kernel may start its prologue now; it
    // waits for this grid's results before its first load (griddepcontrol)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __shared__ __align__(16) uint8_t tile[128][4 * kRepackKb];
    const int64_t groups = (kblocks + kRepackKb - 1) / kRepackKb;
    int64_t rb = static_cast<int64_t>(blockIdx.x) / groups;
    const int64_t g = static_cast<int64_t>(blockIdx.x) - rb * groups;
    const int64_t out_rb = rb;
    const uint8_t *src = sfa;
    int64_t rows = M;
    if (rb >= a_blocks) {
        rb -= a_blocks;
        src = sfb;
        rows = N;
    }
    const int64_t kb0 = g * kRepackKb;
    const int64_t col0 = kb0 * 4;                      // first scale column of this group
    // load: 128 rows x 128 bytes.  16-byte loads when every row starts on a
    // 16-byte boundary (then a 16-byte piece is either wholly inside the row
    // or wholly past it), else byte loads; consecutive threads read
    // consecutive pieces of a row.
    const bool vec = ((reinterpret_cast<uintptr_t>(src) & 15u) == 0) && (k32 % 16 == 0);
    if (vec) {
        constexpr int kPieces = 4 * kRepackKb / 16;
        for (int i = threadIdx.x; i < 128 * kPieces; i += blockDim.x) {
            const int r = i / kPieces;
            const int v = i - r * kPieces;
            const int64_t row = rb * 128 + r;
            const int64_t col = col0 + 16 * v;
            uint4 x = make_uint4(0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
            if (row < rows && col < k32) x = __ldg(reinterpret_cast<const uint4 *>(src + row * k32 + col));
            *reinterpret_cast<uint4 *>(&tile[r][16 * v]) = x;
        }
    } else {
        for (int i = threadIdx.x; i < 128 * 4 * kRepackKb; i += blockDim.x) {
            const int r = i / (4 * kRepackKb);
            const int cidx = i - r * (4 * kRepackKb);
            const int64_t row = rb * 128 + r;
            const int64_t col = col0 + cidx;
            tile[r][cidx] = (row < rows && col < k32) ? src[row * k32 + col] : static_cast<uint8_t>(127);
        }
    }
    __syncthreads();
    // store: chunk j of the group = 32 x 16-byte rows
    const int nkb = static_cast<int>(kblocks - kb0 < kRepackKb ? kblocks - kb0 : kRepackKb);
    for (int i = threadIdx.x; i < nkb * 32; i += blockDim.x) {
        const int j = i / 32;
        const int r = i - j * 32;
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
            w[q] = *reinterpret_cast<const uint32_t *>(&tile[32 * q + r][4 * j]);
        uint4 *dst = reinterpret_cast<uint4 *>(out) + ((out_rb * kblocks + kb0 + j) * 32 + r);
        *dst = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
gemm_mxf8_sm100_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmSF, int64_t sfb_row0, int M, int N, int K,
                       void *C, int64_t ldc, int group_m, DeviceStatus *status, uint64_t timeout_ns) {
    // tmSF views the repacked scales as rows of 512 bytes (128 x 32-bit):
    // row rb * num_kb + kb is the chunk of 128-row block rb at K block kb; the
    // blocks of B start at row sfb_row0.
    constexpr int CG = Cfg::CG;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    const uint32_t base = smem_addr(smem);
    const uint32_t warp = threadIdx.x / 32;
    const uint32_t lane = threadIdx.x % 32;
    const uint32_t rank = (CG == 2) ? cluster_cta_rank() : 0u;

    const uint32_t bar0 = base + Cfg::BAR_OFF;
    auto full_bar = [&](uint32_t s) { return bar0 + 8u * s; };
    auto empty_bar = [&](uint32_t s) { return bar0 + 8u * (Cfg::STAGES + s); };
    const uint32_t tfull_bar = bar0 + 8u * (2 * Cfg::STAGES);
    const uint32_t tempty_bar = tfull_bar + 8u;
    auto sf_full = [&](uint32_t i) { return bar0 + 8u * (2 * Cfg::STAGES + 2 + i); };
    auto sf_empty = [&](uint32_t i) { return bar0 + 8u * (2 * Cfg::STAGES + 2 + Cfg::SF_SLOTS + i); };
    const uint32_t tmem_slot = bar0 + 8u * Cfg::NUM_BARS;
    const uint32_t abort_slot = tmem_slot + 4u;
    volatile uint32_t *tmem_slot_ptr = reinterpret_cast<volatile uint32_t *>(smem + Cfg::BAR_OFF + 8 * Cfg::NUM_BARS);
    volatile uint32_t *abort_flag = tmem_slot_ptr + 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(tfull_bar, 1);
        mbar_init(tempty_bar, Cfg::EPI_WARPS * CG);
        for (int i = 0; i < Cfg::SF_SLOTS; ++i) {
            mbar_init(sf_full(i), 1);
            mbar_init(sf_empty(i), 1);
        }
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_map(&tmA);
        tma_prefetch_map(&tmB);
        tma_prefetch_map(&tmSF);
    }
    if (warp == 1) {
        tmem_alloc<CG>(tmem_slot, Cfg::TMEM_COLS);
        tmem_relinquish<CG>();
    }
    tc_fence_before_sync();
    __syncthreads();
    if constexpr (CG == 2) cluster_sync_all();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot_ptr;

    const int num_m = (M + Cfg::BM - 1) / Cfg::BM;
    const int num_n = (N + Cfg::BN - 1) / Cfg::BN;
    const int num_tiles = num_m * num_n;
    const int num_kb = (K + Cfg::BK - 1) / Cfg::BK;
    const int cluster_id = static_cast<int>(blockIdx.x) / CG;
    const int num_clusters = static_cast<int>(gridDim.x) / CG;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer --
        if (lane == 0) {
            // Launched as a programmatic dependent of the scale repack: the
            // prologue above ran while the repack finished; its chunks (and
            // every earlier write in the stream) are visible after this wait.
            // Without that launch attribute the wait returns at once.
            asm volatile("griddepcontrol.wait;" ::: "memory");
            uint32_t stage = 0, phase = 0;
            bool ok = true;
            for (int tile = cluster_id; ok && tile < num_tiles; tile += num_clusters) {
                int tm, tn;
                raster_tile(tile, num_m, num_n, group_m, tm, tn);
                const int a_rb = tm * CG + static_cast<int>(rank);         // this CTA's 128-row block of A
                const int a_row = a_rb * Cfg::BM_CTA;
                const int b_row = tn * Cfg::BN + static_cast<int>(rank) * Cfg::B_ROWS;
                const int sfa_y = a_rb * num_kb;
                const int sfb_y = static_cast<int>(sfb_row0) + (2 * tn) * num_kb;
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, 2 * timeout_ns)) {
                        record_timeout(status, abort_flag, abort_slot, CG, kRoleProducer * 16 + kBarEmpty);
                        ok = false;
                        break;
                    }
                    const uint32_t a_dst = base + stage * Cfg::STAGE_BYTES;
                    const uint32_t b_dst = a_dst + Cfg::A_BYTES;
                    const uint32_t sfa_dst = b_dst + Cfg::B_BYTES;
                    const uint32_t sfb_dst = sfa_dst + Cfg::SFA_BYTES;
                    const int kx = kb * Cfg::BK;
                    if constexpr (CG == 1) {
                        const uint32_t fb = full_bar(stage);
                        mbar_arrive_expect_tx(fb, Cfg::TX_BYTES);
                        tma_load_2d(a_dst, &tmA, fb, kx, a_row);
                        tma_load_2d(b_dst, &tmB, fb, kx, b_row);
                        tma_load_2d(sfa_dst, &tmSF, fb, 0, sfa_y + kb);
                        tma_load_2d(sfb_dst, &tmSF, fb, 0, sfb_y + kb);
                        tma_load_2d(sfb_dst + Cfg::SF_CHUNK, &tmSF, fb, 0, sfb_y + num_kb + kb);
                    } else {
                        if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), Cfg::TX_BYTES);
                        const uint32_t fb = map_to_cta(full_bar(stage), 0);
                        tma_load_2d_pair(a_dst, &tmA, fb, kx, a_row);
                        tma_load_2d_pair(b_dst, &tmB, fb, kx, b_row);
                        tma_load_2d_pair(sfa_dst, &tmSF, fb, 0, sfa_y + kb);
                        tma_load_2d_pair(sfb_dst, &tmSF, fb, 0, sfb_y + kb);
                        tma_load_2d_pair(sfb_dst + Cfg::SF_CHUNK, &tmSF, fb, 0, sfb_y + num_kb + kb);
                    }
                    if (++stage == Cfg::STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            for (int i = 0; ok && i < Cfg::STAGES; ++i) {
                if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, 2 * timeout_ns)) {
                    record_timeout(status, abort_flag, abort_slot, CG, kRoleProducer * 16 + kBarTail);
                    ok = false;
                }
                if (++stage == Cfg::STAGES) { stage = 0; phase ^= 1u; }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------ MMA issuer (pair leader) --
        if (rank == 0 && lane == 0) {
            uint32_t stage = 0, phase = 0, n = 0;
            bool ok = true;
            int t = 0;
            for (int tile = cluster_id; ok && tile < num_tiles; tile += num_clusters, ++t) {
                if (!mbar_wait(tempty_bar, (static_cast<uint32_t>(t) & 1u) ^ 1u, abort_flag, 3 * timeout_ns)) {
                    record_timeout(status, abort_flag, abort_slot, CG, kRoleMma * 16 + kBarTmemEmpty);
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                for (int kb = 0; kb < num_kb; ++kb) {
                    if (!mbar_wait(full_bar(stage), phase, abort_flag, timeout_ns)) {
                        record_timeout(status, abort_flag, abort_slot, CG, kRoleMma * 16 + kBarFull);
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a0 = base + stage * Cfg::STAGE_BYTES;
                    const uint32_t b0 = a0 + Cfg::A_BYTES;
                    const uint32_t slot = n % Cfg::SF_SLOTS;
                    if (!mbar_wait(sf_full(slot), (n / Cfg::SF_SLOTS) & 1u, abort_flag, timeout_ns)) {
                        record_timeout(status, abort_flag, abort_slot, CG, kRoleMma * 16 + kBarSfFull);
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t sfa_t = tmem_base + Cfg::SF_COL0 + 32u * slot;
                    const uint32_t sfb_t = sfa_t + 16u;
#pragma unroll
                    for (int j = 0; j < Cfg::MMAS; ++j) {
                        const uint32_t idesc = idesc_mxf8_e8m0(Cfg::BM, Cfg::BN, static_cast<uint32_t>(j),
                                                               static_cast<uint32_t>(j));
                        const uint64_t ad = sw128_kmajor_desc(a0 + j * 32);
                        const uint64_t bd = sw128_kmajor_desc(b0 + j * 32);
                        const uint32_t acc = (kb | j) != 0 ? 1u : 0u;
                        if constexpr (CG == 1) mma_mxf8_ss(tmem_base, ad, bd, idesc, sfa_t, sfb_t, acc);
                        else mma_mxf8_ss_pair(tmem_base, ad, bd, idesc, sfa_t, sfb_t, acc);
                    }
                    mma_commit<CG>(empty_bar(stage), 0x3);
                    mma_commit<CG>(sf_empty(slot), 0x1);      // the slot's scales are read
                    ++n;
                    if (++stage == Cfg::STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                mma_commit<CG>(tfull_bar, 0x3);
            }
        }
        __syncwarp();
    } else if (warp == 2 + Cfg::EPI_WARPS) {
        // ---------------------------------- scale copier (pair leader) --
        // tcgen05.cp issued by the MMA thread would run in its issue order,
        // between the MMAs; from this warp the copy of stage s + 1 (or later)
        // is ordered only by the sf_full / sf_empty barriers, so it can run
        // while stage s's MMAs execute.
        if (rank == 0 && lane == 0) {
            uint32_t stage = 0, phase = 0, n = 0;
            bool ok = true;
            for (int tile = cluster_id; ok && tile < num_tiles; tile += num_clusters) {
                for (int kb = 0; kb < num_kb; ++kb, ++n) {
                    const uint32_t slot = n % Cfg::SF_SLOTS;
                    if (!mbar_wait(sf_empty(slot), ((n / Cfg::SF_SLOTS) & 1u) ^ 1u, abort_flag, 2 * timeout_ns)) {
                        record_timeout(status, abort_flag, abort_slot, CG, kRoleSfCopy * 16 + kBarSfEmpty);
                        ok = false;
                        break;
                    }
                    if (!mbar_wait(full_bar(stage), phase, abort_flag, 2 * timeout_ns)) {
                        record_timeout(status, abort_flag, abort_slot, CG, kRoleSfCopy * 16 + kBarFull);
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t sfa_smem = base + stage * Cfg::STAGE_BYTES + Cfg::A_BYTES + Cfg::B_BYTES;
                    const uint32_t sfb_smem = sfa_smem + Cfg::SFA_BYTES;
                    const uint32_t sfa_t = tmem_base + Cfg::SF_COL0 + 32u * slot;
                    const uint32_t sfb_t = sfa_t + 16u;
                    if constexpr (CG == 1) {
                        tmem_cp_32x128b_warpx4(sfa_t, rows16_desc(sfa_smem));
                        tmem_cp_32x128b_warpx4(sfb_t, rows16_desc(sfb_smem));
                        tmem_cp_32x128b_warpx4(sfb_t + 4u, rows16_desc(sfb_smem + Cfg::SF_CHUNK));
                    } else {
                        tmem_cp_32x128b_warpx4_pair(sfa_t, rows16_desc(sfa_smem));
                        tmem_cp_32x128b_warpx4_pair(sfb_t, rows16_desc(sfb_smem));
                        tmem_cp_32x128b_warpx4_pair(sfb_t + 4u, rows16_desc(sfb_smem + Cfg::SF_CHUNK));
                    }
                    mma_commit<CG>(sf_full(slot), 0x1);
                    if (++stage == Cfg::STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            // Tail: the MMA's last releases must land before this CTA exits.
            for (int i = 0; ok && i < Cfg::SF_SLOTS; ++i, ++n) {
                if (!mbar_wait(sf_empty(n % Cfg::SF_SLOTS), ((n / Cfg::SF_SLOTS) & 1u) ^ 1u, abort_flag,
                               2 * timeout_ns)) {
                    record_timeout(status, abort_flag, abort_slot, CG, kRoleSfCopy * 16 + kBarTail);
                    ok = false;
                }
            }
        }
        __syncwarp();
    } else {
        // ----------------------------------------------------- epilogue --
        // TMEM -> registers -> bf16 -> global, 16-byte stores: thread `lane`
        // of warp `sub` owns row 32*sub + lane of this CTA's 128 rows, and
        // each of the two warps on a lane quarter owns half of the columns.
        // The accumulator is single-buffered, so the next tile's MMAs wait for
        // this drain: a warp reads its whole share into registers (as packed
        // bf16, 64 words a thread), hands TMEM back, and only then stores.
        const uint32_t sub = warp & 3u;
        const int half = static_cast<int>(warp - 2) >> 2;
        int t = 0;
        for (int tile = cluster_id; tile < num_tiles; tile += num_clusters, ++t) {
            int tm, tn;
            raster_tile(tile, num_m, num_n, group_m, tm, tn);
            uint32_t ready = 1;
            if (lane == 0 && !mbar_wait(tfull_bar, static_cast<uint32_t>(t) & 1u, abort_flag, 3 * timeout_ns)) {
                record_timeout(status, abort_flag, abort_slot, CG, kRoleEpilogue * 16 + kBarTmemFull);
                ready = 0;
            }
            ready = __shfl_sync(0xffffffffu, ready, 0);
            if (!ready) break;
            tc_fence_after_sync();
            const uint32_t tbase = tmem_base + ((sub * 32u) << 16) + static_cast<uint32_t>(half * Cfg::EPI_COLS);
            const int row = tm * Cfg::BM + static_cast<int>(rank) * Cfg::BM_CTA + static_cast<int>(sub) * 32 +
                            static_cast<int>(lane);
            const int col0 = tn * Cfg::BN + half * Cfg::EPI_COLS;
            uint16_t *crow = reinterpret_cast<uint16_t *>(static_cast<uint8_t *>(C) + static_cast<int64_t>(row) * ldc * 2);
            uint32_t packed[Cfg::EPI_COLS / 2];
            // two 32-column loads per TMEM round trip
#pragma unroll
            for (int g = 0; g < Cfg::EPI_COLS / 32; g += 2) {
                uint32_t v[32], w[32];
                tmem_ld_32x32b_x32(tbase + g * 32, v);
                tmem_ld_32x32b_x32(tbase + g * 32 + 32, w);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    packed[16 * g + i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                    packed[16 * g + 16 + i] = pack_bf16x2(__uint_as_float(w[2 * i]), __uint_as_float(w[2 * i + 1]));
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                if constexpr (CG == 1) mbar_arrive_local(tempty_bar);
                else mbar_arrive_cluster(map_to_cta(tempty_bar, 0));
            }
            if (row >= M) continue;
#pragma unroll
            for (int v = 0; v < Cfg::EPI_COLS / 8; ++v) {    // 8 bf16 = 16 bytes per store
                const int col = col0 + 8 * v;
                if (col >= N) break;
                if (col + 8 <= N) {
                    *reinterpret_cast<uint4 *>(crow + col) =
                        make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        if (col + e < N) crow[col + e] = static_cast<uint16_t>(packed[4 * v + (e >> 1)] >> (16 * (e & 1)));
                }
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if constexpr (CG == 2) cluster_sync_all();
    if (*abort_flag) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000ull) __nanosleep(1000);
    }
    __syncthreads();
    if constexpr (CG == 2) cluster_sync_all();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc<CG>(tmem_base, Cfg::TMEM_COLS);
    }
}

}  // namespace b200
