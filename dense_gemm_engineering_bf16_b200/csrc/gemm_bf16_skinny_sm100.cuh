// Skinny bf16 GEMM for sm_100a (small M): C = A . B with M <= 256.
//
// For a handful of rows of A the product is bound by streaming B from HBM
// (the roofline of "Modern GPU Programming For MLSys - 书籍总结", section 2.2:
// 16 x 8192 x 8192 has an arithmetic intensity of ~16 FLOP/B).  The kernel
// is laid out so that every SM streams an equal share of B:
//
//  * swap A and B: the MMA computes C^T = B . A^T, so 128 rows of B fill the
//    MMA's M = 128 and the (padded) rows of A are its N (16 .. 256, a
//    multiple of 16).  No tensor-core work is spent on padding M up to 128.
//  * stream-K: the iterations (128-row tile of B, 64-wide K block) are
//    flattened and cut into gridDim.x equal contiguous ranges, one per
//    persistent CTA.  A CTA's range crosses at most a few tile boundaries; a
//    tile split across CTAs is finished by whichever contributor arrives
//    last: every contributor writes its fp32 partial to a workspace, bumps
//    the tile's arrival counter, and the last one sums the partials in
//    contributor order (deterministic) and writes C.  A tile owned by one CTA
//    is written directly.  Split-K is in the search space of "GPU 执行模型",
//    section "编译与 autotune".
//
// Roles per CTA (192 threads) as in the square kernel: warp 0 TMA producer,
// warp 1 TMEM owner and MMA issuer, warps 2-5 epilogue (TMEM lane = row of
// B = column n of C).  C rows are written with plain coalesced stores: for a
// fixed m, the 32 lanes of a warp hold 32 consecutive n.
//
// Arrival counters are 64-bit: (epoch << 32) | arrivals.  Each call passes a
// new epoch, so a counter left behind by an earlier, aborted call is simply
// restarted and no reset pass is needed; the last contributor also returns
// its tile's count to zero, so replaying a captured launch (same epoch) works.
#pragma once
#include <cuda_bf16.h>

#include <cstdint>

#include "gemm_bf16_sm100.cuh"
#include "ptx.cuh"

namespace b200 {

template <int MP_, int STAGES_, int OUT_, int KBS_ = 1, bool CSPLIT_ = false>
struct GemmSkinnyCfg {
    // CSPLIT: instead of stream-K over all SMs, a cluster of S = 2 or 4 CTAs
    // per 128-row tile of B, each over its own share of K; the partials meet
    // in shared memory (DSMEM), and the CTA that owns a quarter or half of
    // the tile's columns sums them in member order and writes C.
    static constexpr bool CSPLIT = CSPLIT_;
    static constexpr int MP = MP_;                 // max padded rows of A (MMA N)
    static constexpr int STAGES = STAGES_;
    static constexpr int OUT = OUT_;               // 0: f32 C, 1: bf16 C
    static constexpr int TILE_N = 128;             // rows of B per tile (MMA M)
    static constexpr int BK = 64;                  // K per box (one 128-byte swizzle row)
    static constexpr int KBS = KBS_;               // boxes (64-wide K blocks) per stage
    static constexpr int SK = BK * KBS;            // K per stage, the stream-K iteration unit
    static constexpr int UMMA_K = 16;
    static constexpr int B_BOX = TILE_N * BK * 2;
    static constexpr int A_BOX = MP * BK * 2;
    static constexpr int B_BYTES = KBS * B_BOX;
    static constexpr int A_BYTES = KBS * A_BOX;
    static constexpr int STAGE_BYTES = B_BYTES + A_BYTES;
    static constexpr int TMEM_COLS = pow2_at_least(2 * MP, 32);
    static constexpr int NUM_BARS = 2 * STAGES + 4 + (CSPLIT ? 2 : 0);   // (+ peer_free, rx_full)
    static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
    static constexpr int SMEM_BYTES = 1024 + BAR_OFF + NUM_BARS * 8 + 16;
    static constexpr int THREADS = 192;
    static_assert(MP % 16 == 0 && MP >= 16 && MP <= 256, "MMA N for M = 128");
    static_assert(STAGE_BYTES % 1024 == 0 && A_BOX % 1024 == 0, "swizzle atoms stay 1024-byte aligned");
    static_assert(TMEM_COLS <= 512, "TMEM has 512 columns");
    static_assert(SMEM_BYTES <= 232448, "dynamic shared memory per CTA on sm_100");
    static_assert(!CSPLIT || KBS == 1, "cluster split: one 64-wide K block per stage");
    // the other members' partials of a member's columns (at most 3 x 32 rows
    // of mpad fp32, S = 4) fit in the operand ring
    static_assert(!CSPLIT || 96 * MP * 4 <= STAGES * STAGE_BYTES, "cluster split: receive slots in the ring");
};

// First iteration of CTA c's range when `total` iterations are cut into `g`.
__device__ __forceinline__ int64_t range_begin(int64_t c, int64_t total, int64_t g) {
    return (c * total) / g;
}

// The CTA whose range holds iteration `it`.
__device__ __forceinline__ int64_t range_owner(int64_t it, int64_t total, int64_t g) {
    return ((it + 1) * g + total - 1) / total - 1;
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// C[m][n] = finish(v, C[m][n], bias[n]): the fused epilogue of one element
// (C read only when beta != 0).
template <int OUT>
__device__ __forceinline__ void store_c(void *C, int64_t ldc, int m, int n, float v, const Epilogue &e) {
    const int64_t i = static_cast<int64_t>(m) * ldc + n;
    const float b = e.bias ? __ldg(e.bias + n) : 0.0f;
    if constexpr (OUT == 0) {
        float *c = static_cast<float *>(C);
        c[i] = finish(v, e.beta != 0.0f ? c[i] : 0.0f, b, e);
    } else {
        __nv_bfloat16 *c = static_cast<__nv_bfloat16 *>(C);
        c[i] = __float2bfloat16_rn(finish(v, e.beta != 0.0f ? __bfloat162float(c[i]) : 0.0f, b, e));
    }
}

// The last contributor of a split tile sums the contributors' fp32 partials
// ([m][128] each) in contributor order and writes C rows [0, M) x the tile's
// 128 columns.  Thread t handles four consecutive columns (t % 32) * 4 of
// rows m = 4 j + t / 32.  Each round issues the loads of 4 rows x up to 4
// contributors before summing, so a tile split between up to four CTAs (the
// usual case) costs one round trip to L2 per round; each element is summed
// c_lo, c_lo+1, ... exactly as a sequential loop would.
template <int OUT>
__device__ __forceinline__ void fixup_tile(const float *partials, int64_t slot_elems, int slots_per_cta,
                                           int64_t c_lo, int64_t c_hi, int64_t t, int64_t total, int64_t g,
                                           int64_t kb_per_tile, int M, int N, void *C, int64_t ldc,
                                           uint32_t epi_tid, const Epilogue &epi) {
    constexpr int ROWS = 4;                      // rows per round for this thread
    constexpr int CPR = 4;                       // contributors per round
    const int n4 = static_cast<int>(epi_tid & 31u) * 4;
    const int msub = static_cast<int>(epi_tid >> 5);
    const int n = static_cast<int>(t) * 128 + n4;
    auto slot_ptr = [&](int64_t cc) {
        const int64_t cc_first = ((cc * total) / g) / kb_per_tile;
        return partials + (cc * slots_per_cta + (t - cc_first)) * slot_elems + n4;
    };
    for (int m0 = msub; m0 < M; m0 += 4 * ROWS) {
        float4 acc[ROWS];
#pragma unroll
        for (int r = 0; r < ROWS; ++r) acc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int64_t cc = c_lo; cc <= c_hi; cc += CPR) {
            float4 v[CPR][ROWS];
#pragma unroll
            for (int q = 0; q < CPR; ++q) {
                const bool have = cc + q <= c_hi;
                const float *p = slot_ptr(have ? cc + q : cc);
#pragma unroll
                for (int r = 0; r < ROWS; ++r) {
                    const int m = m0 + 4 * r;
                    v[q][r] = (have && m < M) ? __ldcg(reinterpret_cast<const float4 *>(p + static_cast<int64_t>(m) * 128))
                                              : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
#pragma unroll
            for (int q = 0; q < CPR; ++q) {
                if (cc + q > c_hi) break;
#pragma unroll
                for (int r = 0; r < ROWS; ++r) {
                    acc[r].x += v[q][r].x; acc[r].y += v[q][r].y; acc[r].z += v[q][r].z; acc[r].w += v[q][r].w;
                }
            }
        }
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
            const int m = m0 + 4 * r;
            if (m >= M || n >= N) continue;
            float vals[4] = {acc[r].x, acc[r].y, acc[r].z, acc[r].w};
            if (n + 4 <= N && !epi.identity()) {
                float old[4] = {0.f, 0.f, 0.f, 0.f};
                if (epi.beta != 0.0f) {
                    if constexpr (OUT == 0) {
                        const float4 x = *reinterpret_cast<const float4 *>(static_cast<const float *>(C) +
                                                                           static_cast<int64_t>(m) * ldc + n);
                        old[0] = x.x; old[1] = x.y; old[2] = x.z; old[3] = x.w;
                    } else {
                        const uint2 x = *reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(C) +
                                                                         static_cast<int64_t>(m) * ldc + n);
                        old[0] = __uint_as_float(x.x << 16); old[1] = __uint_as_float(x.x & 0xFFFF0000u);
                        old[2] = __uint_as_float(x.y << 16); old[3] = __uint_as_float(x.y & 0xFFFF0000u);
                    }
                }
                float4 b = make_float4(0.f, 0.f, 0.f, 0.f);
                if (epi.bias) b = __ldg(reinterpret_cast<const float4 *>(epi.bias + n));
                const float bb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) vals[q] = finish(vals[q], old[q], bb[q], epi);
                acc[r] = make_float4(vals[0], vals[1], vals[2], vals[3]);
            }
            if (n + 4 <= N) {
                if constexpr (OUT == 0) {
                    *reinterpret_cast<float4 *>(static_cast<float *>(C) + static_cast<int64_t>(m) * ldc + n) = acc[r];
                } else {
                    const uint32_t lo = pack_bf16x2(vals[0], vals[1]);
                    const uint32_t hi = pack_bf16x2(vals[2], vals[3]);
                    *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(C) + static_cast<int64_t>(m) * ldc + n) =
                        make_uint2(lo, hi);
                }
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (n + q < N) store_c<OUT>(C, ldc, m, n + q, vals[q], epi);
            }
        }
    }
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
gemm_bf16_skinny_sm100_kernel(const __grid_constant__ CUtensorMap tmB,   // B as N x K, box 64 x 64
                              const __grid_constant__ CUtensorMap tmA,   // A as M x K, box 64 x mpad
                              int M, int N, int K, int mpad, void *C, int64_t ldc,
                              float *partials, unsigned long long *counters, int slots_per_cta,
                              uint32_t epoch, DeviceStatus *status, uint64_t timeout_ns,
                              Epilogue epi, uint32_t layout) {
    // B stored K x N arrives as MN-major tiles; A must be stored M x K here.
    const bool b_mn = (layout & kLayoutBMajorN) != 0;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    const uint32_t base = smem_addr(smem);
    const uint32_t warp = threadIdx.x / 32;
    const uint32_t lane = threadIdx.x % 32;
    // cluster split: this CTA's member index and the number of members
    const uint32_t kr = Cfg::CSPLIT ? cluster_cta_rank() : 0u;
    const uint32_t ksplit = Cfg::CSPLIT ? cluster_num_ctas() : 1u;
    const int cluster_ctas = static_cast<int>(ksplit);

    const uint32_t bar0 = base + Cfg::BAR_OFF;
    auto full_bar = [&](uint32_t s) { return bar0 + 8u * s; };
    auto empty_bar = [&](uint32_t s) { return bar0 + 8u * (Cfg::STAGES + s); };
    auto tfull_bar = [&](uint32_t b) { return bar0 + 8u * (2 * Cfg::STAGES + b); };
    auto tempty_bar = [&](uint32_t b) { return bar0 + 8u * (2 * Cfg::STAGES + 2 + b); };
    const uint32_t peer_free_bar = bar0 + 8u * (2 * Cfg::STAGES + 4);   // the others' rings are free
    const uint32_t rx_full_bar = peer_free_bar + 8u;                     // the others' partials are in
    const uint32_t tmem_slot = bar0 + 8u * Cfg::NUM_BARS;
    const uint32_t abort_slot = tmem_slot + 4u;
    volatile uint32_t *tmem_slot_ptr = reinterpret_cast<volatile uint32_t *>(smem + Cfg::BAR_OFF + 8 * Cfg::NUM_BARS);
    volatile uint32_t *abort_flag = tmem_slot_ptr + 1;
    volatile uint32_t *last_flag = tmem_slot_ptr + 2;
    volatile uint32_t *ready_flag = tmem_slot_ptr + 3;

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 4);
        }
        if constexpr (Cfg::CSPLIT) {
            if (ksplit > 1) {
                mbar_init(peer_free_bar, ksplit - 1);                  // one arrival per other member
                mbar_init(rx_full_bar, (ksplit - 1) * (128u / ksplit)); // their threads holding my columns
            }
        }
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_map(&tmA);
        tma_prefetch_map(&tmB);
    }
    if (warp == 1) {
        tmem_alloc<1>(tmem_slot, Cfg::TMEM_COLS);
        tmem_relinquish<1>();
    }
    tc_fence_before_sync();
    __syncthreads();
    if constexpr (Cfg::CSPLIT) cluster_sync_all();   // the others' barriers exist before any remote arrive
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot_ptr;

    // iterations: (tile of 128 rows of B, stage of SK = KBS x 64 K), K fastest
    const int64_t kb_per_tile = (K + Cfg::SK - 1) / Cfg::SK;
    const int64_t tiles = (N + Cfg::TILE_N - 1) / Cfg::TILE_N;
    const int64_t total = tiles * kb_per_tile;
    const int64_t g = gridDim.x;
    const int64_t c = blockIdx.x;
    // stream-K: an equal contiguous share of all iterations per CTA; cluster
    // split: cluster t takes tile t, member kr its share of the tile's K
    const int64_t ctile = static_cast<int64_t>(blockIdx.x) / ksplit;
    const int64_t it_begin = Cfg::CSPLIT ? ctile * kb_per_tile + (static_cast<int64_t>(kr) * kb_per_tile) / ksplit
                                         : range_begin(c, total, g);
    const int64_t it_end = Cfg::CSPLIT ? ctile * kb_per_tile + (static_cast<int64_t>(kr + 1) * kb_per_tile) / ksplit
                                       : range_begin(c + 1, total, g);
    const int64_t first_tile = Cfg::CSPLIT ? ctile : it_begin / kb_per_tile;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer --
        if (lane == 0) {
            const uint32_t box_tx = static_cast<uint32_t>(Cfg::B_BOX + mpad * Cfg::BK * 2);
            const int k_boxes = (K + Cfg::BK - 1) / Cfg::BK;
            // Each byte of B is read once: evict_first keeps the stream from
            // displacing A and the split-tile partials in L2 (measured: 38.9
            // vs 43.1 us per 16 x 8192 x 8192 step).
            const uint64_t stream_b = l2_policy_evict_first();
            uint32_t stage = 0, phase = 0;
            bool ok = true;
            for (int64_t it = it_begin; it < it_end; ++it) {
                const int t = static_cast<int>(it / kb_per_tile);
                const int kb = static_cast<int>(it - static_cast<int64_t>(t) * kb_per_tile);
                if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, 2 * timeout_ns)) {
                    record_timeout(status, abort_flag, abort_slot, cluster_ctas, kRoleProducer * 16 + kBarEmpty);
                    ok = false;
                    break;
                }
                const uint32_t b_dst = base + stage * Cfg::STAGE_BYTES;
                const uint32_t a_dst = b_dst + Cfg::B_BYTES;
                // the stage's boxes back to back: for every row of B, up to
                // KBS adjacent 128-byte pieces are requested close together;
                // boxes wholly past K (the last stage of a tile) are skipped
                const int nbox = min(Cfg::KBS, k_boxes - kb * Cfg::KBS);
                mbar_arrive_expect_tx(full_bar(stage), static_cast<uint32_t>(nbox) * box_tx);
                // K-major B arrives as two 64-row boxes per 128-row tile (measured:
                // 35.3 against 36.1 us at 16 x 8192 x 8192 with one 128-row box)
                for (int j = 0; j < nbox; ++j) {
                    const int kx = (kb * Cfg::KBS + j) * Cfg::BK;
                    if (b_mn) {
                        load_operand_tile<1, true>(b_dst + j * Cfg::B_BOX, &tmB, full_bar(stage), kx,
                                                   t * Cfg::TILE_N, Cfg::TILE_N, true, stream_b);
                    } else {
                        tma_load_2d_hint(b_dst + j * Cfg::B_BOX, &tmB, full_bar(stage), kx, t * Cfg::TILE_N, stream_b);
                        tma_load_2d_hint(b_dst + j * Cfg::B_BOX + Cfg::B_BOX / 2, &tmB, full_bar(stage), kx,
                                         t * Cfg::TILE_N + Cfg::TILE_N / 2, stream_b);
                    }
                }
                for (int j = 0; j < nbox; ++j)
                    tma_load_2d(a_dst + j * Cfg::A_BOX, &tmA, full_bar(stage), (kb * Cfg::KBS + j) * Cfg::BK, 0);
                if (++stage == Cfg::STAGES) { stage = 0; phase ^= 1u; }
            }
            for (int i = 0; ok && i < Cfg::STAGES; ++i) {
                if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, 2 * timeout_ns)) {
                    record_timeout(status, abort_flag, abort_slot, cluster_ctas, kRoleProducer * 16 + kBarTail);
                    ok = false;
                }
                if (++stage == Cfg::STAGES) { stage = 0; phase ^= 1u; }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // --------------------------------------------------- MMA issuer --
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(Cfg::TILE_N, mpad, b_mn ? 1u : 0u, 0u);
            const int k_boxes = (K + Cfg::BK - 1) / Cfg::BK;
            uint32_t stage = 0, phase = 0;
            bool ok = true;
            int seg = 0;
            int64_t it = it_begin;
            while (ok && it < it_end) {
                const int64_t t = it / kb_per_tile;
                const int64_t seg_end = min(it_end, (t + 1) * kb_per_tile);
                const uint32_t buf = static_cast<uint32_t>(seg) & 1u;
                if (!mbar_wait(tempty_bar(buf), ((static_cast<uint32_t>(seg) >> 1) & 1u) ^ 1u, abort_flag,
                               3 * timeout_ns)) {
                    record_timeout(status, abort_flag, abort_slot, cluster_ctas, kRoleMma * 16 + kBarTmemEmpty);
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + buf * Cfg::MP;
                for (int64_t j = it; j < seg_end; ++j) {
                    if (!mbar_wait(full_bar(stage), phase, abort_flag, timeout_ns)) {
                        record_timeout(status, abort_flag, abort_slot, cluster_ctas, kRoleMma * 16 + kBarFull);
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t bs = base + stage * Cfg::STAGE_BYTES;
                    const uint32_t as = bs + Cfg::B_BYTES;
                    const int nbox = min(Cfg::KBS, k_boxes - static_cast<int>(j - t * kb_per_tile) * Cfg::KBS);
                    for (int q = 0; q < nbox; ++q) {
                        const uint32_t b0 = bs + q * Cfg::B_BOX;
                        const uint32_t a0 = as + q * Cfg::A_BOX;
#pragma unroll
                        for (int kk = 0; kk < Cfg::BK / Cfg::UMMA_K; ++kk) {
                            mma_bf16_ss<1>(d_tmem, operand_desc(b0, kk, b_mn), sw128_kmajor_desc(a0 + kk * 32),
                                           idesc, (j != it || q != 0 || kk != 0) ? 1u : 0u);
                        }
                    }
                    mma_commit<1>(empty_bar(stage), 0);
                    if (++stage == Cfg::STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                mma_commit<1>(tfull_bar(buf), 0);
                it = seg_end;
                ++seg;
            }
        }
        __syncwarp();
    } else {
        // ----------------------------------------------------- epilogue --
        const uint32_t sub = warp & 3u;
        const int n_local = static_cast<int>(sub * 32u + lane);
        const uint32_t epi_tid = threadIdx.x - 64u;          // 0..127
        const int64_t slot_elems = static_cast<int64_t>(Cfg::TILE_N) * Cfg::MP;
        int seg = 0;
        int64_t it = it_begin;
        if constexpr (Cfg::CSPLIT) {
            // ---- cluster split: member kr holds the fp32 partial of its
            // share of K (none: zeros).  Each warp's 32 columns of C belong to
            // member owner = its lane quarter / (4 / S): the other members'
            // warps on those columns send their partials (all mpad rows) to
            // a slot of the owner's operand ring, and the owner's warp adds
            // the S partials in member order and writes C.
            const uint32_t S = ksplit;
            const bool has_k = it_end > it_begin;
            bool ok = true;
            if (has_k) {
                if (epi_tid == 0) {
                    uint32_t r = 1;
                    if (!mbar_wait(tfull_bar(0), 0, abort_flag, 3 * timeout_ns)) {
                        record_timeout(status, abort_flag, abort_slot, cluster_ctas, kRoleEpilogue * 16 + kBarTmemFull);
                        r = 0;
                    }
                    *ready_flag = r;
                }
                named_barrier_sync(1, 128);
                ok = *ready_flag != 0;
                tc_fence_after_sync();
            }
            const uint32_t lanes_per = 128u / S;
            const uint32_t owner = (sub * 32u) / lanes_per;
            const uint32_t tbase = tmem_base + ((sub * 32u) << 16);          // accumulator buffer 0
            const uint32_t row_bytes = static_cast<uint32_t>(mpad) * 4u;
            const uint32_t slot_bytes = lanes_per * row_bytes;
            const uint32_t r_in = sub * 32u + lane - owner * lanes_per;      // row in the owner's slots
            // 16-byte pieces of a row (mpad / 4 of them, a multiple of 4)
            // rotated within groups of four by the row: fewer bank conflicts
            auto piece_addr = [&](uint32_t row_base, int m0, int p) {
                return row_base + (((static_cast<uint32_t>(m0 / 4 + p)) ^ (lane & 3u)) << 4);
            };
            auto load16 = [&](int m0, uint32_t (&v)[16]) {
                if (has_k) {
                    tmem_ld_32x32b_x16(tbase + static_cast<uint32_t>(m0), v);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = 0u;
                }
            };
            if (ok && S > 1) {
                // this CTA's MMAs are done: its ring may take the others' partials
                if (epi_tid == 0)
                    for (uint32_t j = 0; j < S; ++j)
                        if (j != kr) mbar_arrive_cluster(map_to_cta(peer_free_bar, j));
                uint32_t wok = 1;
                if (owner != kr) {
                    if (lane == 0 && !mbar_wait(peer_free_bar, 0, abort_flag, 3 * timeout_ns)) {
                        record_timeout(status, abort_flag, abort_slot, cluster_ctas, kRoleEpilogue * 16 + kBarPeerFree);
                        wok = 0;
                    }
                    wok = __shfl_sync(0xffffffffu, wok, 0);
                    __syncwarp();   // lane 0's acquire orders every lane's accesses that follow
                    if (wok) {
                        const uint32_t slot = kr < owner ? kr : kr - 1u;
                        const uint32_t dst_row = map_to_cta(base + slot * slot_bytes + r_in * row_bytes, owner);
                        for (int m0 = 0; m0 < mpad; m0 += 16) {
                            uint32_t v[16];
                            load16(m0, v);
#pragma unroll
                            for (int p = 0; p < 4; ++p)
                                store_cluster_v4(piece_addr(dst_row, m0, p), v[4 * p], v[4 * p + 1], v[4 * p + 2],
                                                 v[4 * p + 3]);
                        }
                        mbar_arrive_cluster(map_to_cta(rx_full_bar, owner));   // release: the stores come first
                    }
                } else {
                    if (lane == 0 && !mbar_wait(rx_full_bar, 0, abort_flag, 3 * timeout_ns)) {
                        record_timeout(status, abort_flag, abort_slot, cluster_ctas, kRoleEpilogue * 16 + kBarRxFull);
                        wok = 0;
                    }
                    wok = __shfl_sync(0xffffffffu, wok, 0);
                    __syncwarp();   // lane 0's acquire orders every lane's accesses that follow
                }
                ok = wok != 0;
            }
            if (ok && owner == kr) {
                const int n = static_cast<int>(first_tile) * Cfg::TILE_N + n_local;
                for (int m0 = 0; m0 < mpad; m0 += 16) {
                    uint32_t own[16];
                    load16(m0, own);
                    float acc[16];
                    for (uint32_t mm = 0; mm < S; ++mm) {
                        uint32_t x[16];
                        if (mm == kr) {
#pragma unroll
                            for (int i = 0; i < 16; ++i) x[i] = own[i];
                        } else {
                            const uint32_t slot = mm < kr ? mm : mm - 1u;
                            const uint32_t src_row = base + slot * slot_bytes + r_in * row_bytes;
#pragma unroll
                            for (int p = 0; p < 4; ++p)
                                ld_shared_v4(piece_addr(src_row, m0, p), x[4 * p], x[4 * p + 1], x[4 * p + 2],
                                             x[4 * p + 3]);
                        }
#pragma unroll
                        for (int i = 0; i < 16; ++i) acc[i] = mm == 0 ? __uint_as_float(x[i]) : acc[i] + __uint_as_float(x[i]);
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int m = m0 + i;
                        if (m < M && n < N) store_c<Cfg::OUT>(C, ldc, m, n, acc[i], epi);
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_local(tempty_bar(0));
            it = it_end;                              // one tile per cluster: nothing further
        }
        while (it < it_end) {
            const int64_t t = it / kb_per_tile;
            const int64_t seg_end = min(it_end, (t + 1) * kb_per_tile);
            const uint32_t buf = static_cast<uint32_t>(seg) & 1u;
            const int64_t c_lo = range_owner(t * kb_per_tile, total, g);
            const int64_t c_hi = range_owner((t + 1) * kb_per_tile - 1, total, g);
            const bool shared_tile = c_hi > c_lo;
            // One thread waits; all 128 epilogue threads take its result, so
            // they stay in step for the named barriers below.
            if (epi_tid == 0) {
                uint32_t ok = 1;
                if (!mbar_wait(tfull_bar(buf), (static_cast<uint32_t>(seg) >> 1) & 1u, abort_flag, 3 * timeout_ns)) {
                    record_timeout(status, abort_flag, abort_slot, cluster_ctas, kRoleEpilogue * 16 + kBarTmemFull);
                    ok = 0;
                }
                *ready_flag = ok;
            }
            named_barrier_sync(1, 128);
            if (!*ready_flag) break;
            tc_fence_after_sync();
            const int n = static_cast<int>(t) * Cfg::TILE_N + n_local;
            float *my_partial = partials + (c * slots_per_cta + (t - first_tile)) * slot_elems;
            const uint32_t tbase = tmem_base + ((sub * 32u) << 16) + buf * Cfg::MP;
            for (int m0 = 0; m0 < mpad; m0 += 16) {
                uint32_t v[16];
                tmem_ld_32x32b_x16(tbase + static_cast<uint32_t>(m0), v);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int m = m0 + i;
                    if (m < M) {
                        const float x = __uint_as_float(v[i]);
                        if (shared_tile) my_partial[static_cast<int64_t>(m) * Cfg::TILE_N + n_local] = x;
                        else if (n < N) store_c<Cfg::OUT>(C, ldc, m, n, x, epi);
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_local(tempty_bar(buf));

            if (shared_tile) {
                // Publish this partial, count the arrival; the last of the
                // tile's contributors sums all partials in contributor order.
                // The barrier orders the 128 threads' partial stores before
                // thread 0's gpu-scope fence, which (being cumulative) makes
                // them visible before its counter update.
                named_barrier_sync(1, 128);
                if (epi_tid == 0) {
                    __threadfence();
                    unsigned long long *ctr = counters + t;
                    const unsigned long long tag = static_cast<unsigned long long>(epoch) << 32;
                    unsigned long long old = *reinterpret_cast<volatile unsigned long long *>(ctr), seen;
                    unsigned long long want;
                    do {
                        seen = old;
                        want = ((seen & 0xFFFFFFFF00000000ull) == tag) ? seen + 1ull : (tag | 1ull);
                        old = atomicCAS(ctr, seen, want);
                    } while (old != seen);
                    *last_flag = ((want & 0xFFFFFFFFull) == static_cast<unsigned long long>(c_hi - c_lo + 1)) ? 1u : 0u;
                }
                named_barrier_sync(1, 128);
                if (*last_flag) {
                    __threadfence();
                    fixup_tile<Cfg::OUT>(partials, slot_elems, slots_per_cta, c_lo, c_hi, t, total, g,
                                         kb_per_tile, M, N, C, ldc, epi_tid, epi);
                    // every contributor has arrived: leave the counter at zero
                    // arrivals so a replay of this launch (same epoch, e.g.
                    // from a CUDA graph) starts from a clean count
                    if (epi_tid == 0) counters[t] = static_cast<unsigned long long>(epoch) << 32;
                }
                named_barrier_sync(1, 128);
            }
            it = seg_end;
            ++seg;
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if constexpr (Cfg::CSPLIT) cluster_sync_all();
    if (*abort_flag) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000ull) __nanosleep(1000);
    }
    __syncthreads();
    if constexpr (Cfg::CSPLIT) cluster_sync_all();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc<1>(tmem_base, Cfg::TMEM_COLS);
    }
}

}  // namespace b200
