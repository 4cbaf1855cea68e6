// Persistent, warp-specialised bf16 GEMM for sm_100a:  C = A . B
//
// The construction follows part III of "Modern GPU Programming For MLSys -
// 书籍总结" (omica.com.cn): a 128 x N output tile (step 1), K-loop
// accumulation (step 2), tiles spread over CTAs (step 3), TMA loads (step 4),
// a multi-stage shared-memory ring (step 5), a persistent kernel walking a
// tile schedule (step 6), warp specialisation into TMA producer / MMA issuer
// / write-back (step 7) and, for CG == 2, a CTA pair running one
// cta_group::2 MMA over both CTAs' shared memory with a 256-row tile (step 8).
// With CONSUMERS == 2 a second MMA consumer stacks another 256 rows on the
// same B k-tiles, a 512 x 256 pair tile (step 9): both accumulators fill
// TMEM, so it holds one tile at a time instead of two.
//
// Per CTA (192 threads):
//   warp 0      TMA producer: waits empty[s], loads the A and B k-tiles of
//               stage s (128-byte swizzle), completion counted in bytes on
//               the pair leader's full[s].
//   warp 1      TMEM owner (alloc / dealloc) and, in the pair leader only, the
//               MMA issuer: waits full[s], issues BK/16 tcgen05.mma per
//               consumer into its TMEM accumulator, commits to empty[s] (both
//               CTAs); after the last k-tile of a tile commits to
//               tmem_full[b].
//   warps 2-5   epilogue: waits tmem_full[b], tcgen05.ld 32 rows x 32 columns
//               per warp, converts, writes a swizzled staging buffer, and TMA-
//               stores it; releases tmem_empty[b] (pair leader's barrier)
//               once the accumulators are read.  With one consumer TMEM holds
//               two tiles (2 x BN columns), so tile i+1's main loop runs while
//               tile i drains; with two, the drain is the MMA's only stall.
//
//   warp 6      (CLC builds only) scheduler, in the pair leader: claims tiles
//               of clusters that have not started with
//               clusterlaunchcontrol.try_cancel ("Modern GPU Programming For
//               MLSys - 书籍总结", section 2.9: fast CTAs pull more work instead
//               of idling) and hands the tile id to every role of both CTAs
//               through a 2-deep shared-memory ring.
//
// Cluster split-K (SPLITK, one-CTA tiles): a cluster of S = 2, 4 or 8 CTAs
// owns one tile, member r accumulating K blocks [r kb / S, (r+1) kb / S).
// Once its MMAs are done, each member tells the others that its operand
// ring is free.  It then sends column slice j of its fp32 partial into a
// slot of member j's ring, through distributed shared memory, with a
// cluster-scope release arrive on j's rx_full.  Member j adds the S partials
// of its slice in member order and writes them to C through the usual store
// path.  The split-K schedule of the pages' autotune search space ("GPU
// 执行模型", section "编译与 autotune"), with the reduction on chip: no
// workspace, no atomics, and a fixed summation order.
//
// Narrow tail (TAIL: one consumer, static or CLC schedule, K-major B): when
// the tiles left for a last wave would occupy at most half of the
// co-resident clusters, each of them runs as two units of BN / 2 columns
// (an MMA of N = BN / 2 over half of the B rows), so the clusters that would
// have idled take the other halves.  This is the wave-tail entry of the
// pages' autotune search space ("GPU 执行模型", section "编译与 autotune":
// tile shape and persistent strategy), without a reduction: each half is a
// whole block of C.
//
// Operands may be K-major (A as M x K, B as N x K) or MN-major (A as K x M,
// B as K x N): MN-major tiles arrive as 64-wide boxes and the MMA reads them
// through MN-major descriptors.  The epilogue computes
// act(alpha * A.B + beta * C + bias) in fp32 before the output rounding
// (epilogue.cuh; C read only when beta != 0).
//
// Tails: TMA loads zero-fill outside [0,K) x [0,M) / [0,N) element by
// element.  TMA stores clip rows exactly but write whole 16-byte granules
// along a row, so C's tensor map covers only the columns [0, n_tma) that end
// on a granule boundary; the last < 16 bytes of each row ([n_tma, N)) are
// written with plain predicated stores.  Every mbarrier wait is bounded.
#pragma once
#include <cuda_bf16.h>

#include <cstdint>
#include <type_traits>

#include "epilogue.cuh"
#include "ptx.cuh"

namespace b200 {

// Device status block (global memory, one per device).  code != 0 records
// the first expired wait; the host reads and clears it.
struct DeviceStatus {
    uint32_t code;
    int32_t where;
    int32_t block;
    uint32_t pad;
};

constexpr uint32_t kStatusTimeout = 6;   // == GEMM_ERR_TIMEOUT

// Test-only fault injection (host side: B200GEMM_INJECT_TIMEOUT): CTA 0 skips
// its first k-tile, leaving that stage's full barrier unarmed, so the MMA
// warp's bounded wait expires and the abort path runs.  Nothing faults.
constexpr uint32_t kInjectDropFirstStage = 1u;

enum : int { kRoleProducer = 1, kRoleMma = 2, kRoleEpilogue = 3, kRoleScheduler = 4 };
enum : int { kBarFull = 1, kBarEmpty = 2, kBarTmemFull = 3, kBarTmemEmpty = 4, kBarTail = 5, kBarSched = 6,
             kBarClc = 7, kBarPeerFree = 10, kBarRxFull = 11 };

__host__ __device__ constexpr int pow2_at_least(int v, int lo) {
    int p = lo;
    while (p < v) p *= 2;
    return p;
}

// More copies of C for the row-sharded GEMM with its all-gather fused in:
// the epilogue stores every finished chunk of the slab to up to kMaxPeerC
// further destinations (other GPUs' C through their mapped pointers), each
// described by a tensor map of the slab in that C and the slab's base
// pointer there (for the plain stores of each row's ragged end).
constexpr int kMaxPeerC = 7;
struct PeerC {
    CUtensorMap map[kMaxPeerC];
    void *base[kMaxPeerC];
    int count;
};
struct NoPeerC {};

template <int CG_, int BN_, int STAGES_, int OUT_, bool CLC_ = false, int CONSUMERS_ = 1, bool SK_ = false,
          bool PEERS_ = false, bool SPLITK_ = false, bool TAIL_ = false>
struct GemmBf16Cfg {
    static constexpr bool CLC = CLC_;              // tiles from Cluster Launch Control, not a fixed stride
    // Stream-K: the (tile, K block) iterations are cut into one contiguous
    // range per cluster; a tile split between clusters is summed from fp32
    // partials by the last of its contributors, in contributor order.
    static constexpr bool SK = SK_;
    // PEERS: every chunk of C is also stored to the destinations of a PeerC
    static constexpr bool PEERS = PEERS_;
    // SPLITK: cluster split-K.  The S CTAs of a cluster (S = 2, 4 or 8, the
    // launch's cluster size) compute one tile together, each over its own
    // contiguous share of the K blocks.  Member j then sums column slice j
    // of the tile from every member's fp32 partial, in member order, the
    // partials crossing between the CTAs' shared memories (DSMEM).
    static constexpr bool SPLITK = SPLITK_;
    using PeerArg = std::conditional_t<PEERS_, PeerC, NoPeerC>;
    static constexpr int CG = CG_;                 // CTAs per tile (cta_group)
    static constexpr int BN = BN_;                 // tile N == MMA N
    static constexpr int STAGES = STAGES_;         // shared-memory ring depth
    static constexpr int OUT = OUT_;               // 0: f32 C, 1: bf16 C
    // MMA consumers per tile: 2 stacks two MMA-M row blocks in one tile that
    // share every B k-tile (a 512 x 256 pair tile), each with its own TMEM
    // accumulator; TMEM then holds no second tile, so it is single-buffered.
    static constexpr int CONSUMERS = CONSUMERS_;
    static constexpr int BM_CTA = 128;             // accumulator rows per CTA and consumer (TMEM lanes)
    static constexpr int BM_MMA = 128 * CG;        // MMA M
    static constexpr int BM = BM_MMA * CONSUMERS;  // tile M
    static constexpr int BK = 64;                  // 64 bf16 = one 128-byte swizzle row
    static constexpr int UMMA_K = 16;              // K per tcgen05.mma (kind::f16)
    static constexpr int B_ROWS = BN / CG;         // B rows this CTA loads per k-tile
    static constexpr int A_PART_BYTES = BM_CTA * BK * 2;     // one consumer's A rows of this CTA
    static constexpr int A_BYTES = CONSUMERS * A_PART_BYTES;
    static constexpr int B_BYTES = B_ROWS * BK * 2;
    static constexpr int ACC_BUFS = CONSUMERS == 1 ? 2 : 1;  // tiles held in TMEM at once
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int TX_BYTES = STAGE_BYTES * CG;   // bytes landing on the leader's full[s]
    static constexpr int EPI_COLS = OUT == 0 ? 32 : 64; // columns in one 128-byte staged row
    static constexpr int EPI_CHUNKS = BN / EPI_COLS;
    static constexpr int EPI_BUF = 32 * 128;       // one warp's 32 rows x 128 bytes
    static constexpr int EPI_BYTES = 4 * 2 * EPI_BUF;
    static constexpr int TMEM_COLS = pow2_at_least(ACC_BUFS * CONSUMERS * BN, 32);
    // full[S], empty[S], tmem_full[2], tmem_empty[2] (+ clc[2], sched_full[2], sched_empty[2])
    // (+ split-K: peer_free, rx_full)
    static constexpr int NUM_BARS = 2 * STAGES + 4 + (CLC ? 6 : 0) + (SPLITK ? 2 : 0);
    static constexpr int BAR_OFF = STAGES * STAGE_BYTES + EPI_BYTES;
    // after the barriers: TMEM address, abort flag, 2 tile ids, 2 CLC answers
    static constexpr int SMEM_BYTES = 1024 + BAR_OFF + NUM_BARS * 8 + 64;
    static constexpr int THREADS = CLC ? 224 : 192;        // + one scheduler warp
    // Narrow tail: when the last wave of tiles would fill at most half of the
    // co-resident clusters, each of its tiles may run as two half-width units
    // (BN / 2 columns each) on two clusters, so that every cluster gets work.
    // TAIL_OK: this tile has such a twin (Tail), a separate instantiation
    // launched only when the tail splits, so that whole-tile launches run
    // code without the half-unit logic.
    static constexpr bool TAIL_OK = CONSUMERS == 1 && !SK && !SPLITK && !PEERS && (BN / 2) % EPI_COLS == 0 &&
                                    (B_ROWS / 2) % 8 == 0;
    static constexpr bool TAIL = TAIL_;
    using Tail = GemmBf16Cfg<CG_, BN_, STAGES_, OUT_, CLC_, CONSUMERS_, SK_, PEERS_, SPLITK_, true>;
    static constexpr int SCHED_CONSUMERS = CG == 1 ? 6 : 11;  // arrivals that free a tile slot

    static_assert(CG == 1 || CG == 2, "cta_group is 1 or 2");
    static_assert(CONSUMERS == 1 || CONSUMERS == 2, "one or two MMA consumers");
    static_assert(!SK || (!CLC && CONSUMERS == 1 && BN % 4 == 0), "stream-K: static schedule, one consumer");
    static_assert(!PEERS || !SK, "a stream-K fix-up writes C with plain stores to one C only");
    static_assert(!SPLITK || (CG == 1 && !CLC && CONSUMERS == 1 && !SK && !PEERS),
                  "cluster split-K: one-CTA tiles, one tile per cluster, one C");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N: multiple of 16 in [16, 256]");
    static_assert(B_ROWS % 8 == 0 && B_ROWS <= 256, "TMA box rows <= 256, whole 8-row swizzle atoms");
    static_assert(BN % EPI_COLS == 0, "epilogue chunks cover the tile");
    static_assert(TMEM_COLS <= 512, "TMEM has 512 columns");
    static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "swizzle atoms stay 1024-byte aligned");
    static_assert(SMEM_BYTES <= 232448, "dynamic shared memory per CTA on sm_100");
    static_assert(SMEM_BYTES < (1 << 18), "descriptor start addresses (18 bits) cannot carry");
    static_assert(!TAIL || TAIL_OK, "narrow tail: one consumer, whole-tile schedule, whole store chunks per half");
};

// Tile index -> (tile row, tile column), grouped along M so that CTAs
// running at the same time share A row-panels and B column-panels in L2.
__device__ __forceinline__ void raster_tile(int tile, int num_m, int num_n, int group_m,
                                            int &tm, int &tn) {
    const int group_size = group_m * num_n;
    const int group = tile / group_size;
    const int first_m = group * group_m;
    const int rows = min(group_m, num_m - first_m);
    const int local = tile - group * group_size;
    tm = first_m + local % rows;
    tn = local / rows;
}

// A bounded wait failed.  If it failed because this CTA was already told to
// abort, someone else has recorded the cause: just leave.  Otherwise record
// the first expired wait of the grid (role, barrier, CTA), then tell this CTA
// and the other `cluster_ctas - 1` CTAs of its cluster to abort.
__device__ __forceinline__ void record_timeout(DeviceStatus *status, volatile uint32_t *abort_flag,
                                               uint32_t abort_smem, int cluster_ctas, int where) {
    if (*abort_flag) return;
    if (atomicCAS(&status->code, 0u, kStatusTimeout) == 0u) {
        status->where = where;
        status->block = static_cast<int32_t>(blockIdx.x);
        __threadfence();
    }
    *abort_flag = 1u;
    if (cluster_ctas > 1) {
        const uint32_t me = cluster_cta_rank();
        for (uint32_t r = 0; r < static_cast<uint32_t>(cluster_ctas); ++r)
            if (r != me) store_cluster_u32(map_to_cta(abort_smem, r), 1u);
    }
}

// Operand layouts in global memory (kernel `layout` word).
constexpr uint32_t kLayoutAMajorM = 1u;   // A stored K x M: a(i,k) at A[k*lda + i]
constexpr uint32_t kLayoutBMajorN = 2u;   // B stored K x N: b(k,j) at B[k*ldb + j]

// One k-tile of an operand into shared memory.  K-major: one box of 64 (K)
// x rows.  MN-major: rows / 64 boxes of 64 (MN) x 64 (K), 8 KB apart (the
// layout sw128_mnmajor_desc describes).  Completion counts on `bar`.
// HINT: the loads carry the L2 policy `policy` (else the default policy).
template <int CG, bool HINT = false>
__device__ __forceinline__ void load_one_box(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y,
                                             uint64_t policy) {
    if constexpr (HINT) {
        if constexpr (CG == 1) tma_load_2d_hint(dst, map, bar, x, y, policy);
        else tma_load_2d_pair_hint(dst, map, bar, x, y, policy);
    } else {
        (void)policy;
        if constexpr (CG == 1) tma_load_2d(dst, map, bar, x, y);
        else tma_load_2d_pair(dst, map, bar, x, y);
    }
}

template <int CG, bool HINT = false>
__device__ __forceinline__ void load_operand_tile(uint32_t dst, const CUtensorMap *map, uint32_t bar, int kx,
                                                  int row, int rows, bool mn, uint64_t policy = 0) {
    if (!mn) {
        load_one_box<CG, HINT>(dst, map, bar, kx, row, policy);
        return;
    }
    for (int h = 0; h < rows / 64; ++h) load_one_box<CG, HINT>(dst + 8192u * h, map, bar, row + 64 * h, kx, policy);
}

// Descriptor of K step kk (16 elements) of an operand tile at `base`.
__device__ __forceinline__ uint64_t operand_desc(uint32_t base, int kk, bool mn) {
    return mn ? sw128_mnmajor_desc(base + 2048u * kk) : sw128_kmajor_desc(base + 32u * kk);
}

__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// C[row][col .. col + 3] = finish(v, C_old, bias) for the columns below N.
template <int OUT>
__device__ __forceinline__ void store4_c(void *C, int64_t ldc, int row, int col, float (&v)[4], int N,
                                         const Epilogue &epi) {
    const int64_t i = static_cast<int64_t>(row) * ldc + col;
    if (!epi.identity()) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (col + q >= N) break;
            float old = 0.0f;
            if (epi.beta != 0.0f) {
                if constexpr (OUT == 0) old = static_cast<const float *>(C)[i + q];
                else old = __bfloat162float(static_cast<const __nv_bfloat16 *>(C)[i + q]);
            }
            v[q] = finish(v[q], old, epi.bias ? __ldg(epi.bias + col + q) : 0.0f, epi);
        }
    }
    if (col + 4 <= N) {
        if constexpr (OUT == 0) {
            *reinterpret_cast<float4 *>(static_cast<float *>(C) + i) = make_float4(v[0], v[1], v[2], v[3]);
        } else {
            *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(C) + i) =
                make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
        }
    } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (col + q >= N) break;
            if constexpr (OUT == 0) static_cast<float *>(C)[i + q] = v[q];
            else static_cast<__nv_bfloat16 *>(C)[i + q] = __float2bfloat16_rn(v[q]);
        }
    }
}

// Stream-K fix-up by the last contributor of a split tile, for this CTA's
// 128 rows: C rows [row0, row0 + 128) x columns [col0, col0 + BN) = the sum
// of the contributors' fp32 partials ([128][BN] each, `part(cc)`) in
// contributor order c_lo, c_lo + 1, ..., then the epilogue.  128 threads;
// thread `tid` owns four consecutive columns and every (128 / (BN / 4))-th
// row; each round keeps 8 rows x 2 contributors of float4 loads in flight.
template <int OUT, int BN, class PartFn>
__device__ __forceinline__ void sk_fixup(PartFn part, int64_t c_lo, int64_t c_hi, int row0, int col0, int M,
                                         int N, void *C, int64_t ldc, uint32_t tid, const Epilogue &epi) {
    constexpr int TPR = BN / 4;          // threads per row
    constexpr int RPP = 128 / TPR;       // rows per pass of the 128 threads
    constexpr int ROWS = 8;
    static_assert(128 % TPR == 0 && (128 / RPP) % ROWS == 0, "fix-up thread layout");
    const int c4 = static_cast<int>(tid % TPR) * 4;
    const int r_first = static_cast<int>(tid / TPR);
    const int col = col0 + c4;
    for (int rb = 0; rb < 128 / RPP; rb += ROWS) {
        float4 acc[ROWS];
#pragma unroll
        for (int r = 0; r < ROWS; ++r) acc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int64_t cc = c_lo; cc <= c_hi; cc += 2) {
            const bool two = cc + 1 <= c_hi;
            const float *p0 = part(cc) + c4;
            const float *p1 = two ? part(cc + 1) + c4 : p0;
            float4 v0[ROWS], v1[ROWS];
#pragma unroll
            for (int r = 0; r < ROWS; ++r) {
                const int lr = r_first + RPP * (rb + r);
                v0[r] = __ldcg(reinterpret_cast<const float4 *>(p0 + static_cast<int64_t>(lr) * BN));
                v1[r] = two ? __ldcg(reinterpret_cast<const float4 *>(p1 + static_cast<int64_t>(lr) * BN))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int r = 0; r < ROWS; ++r) {
                acc[r].x += v0[r].x; acc[r].y += v0[r].y; acc[r].z += v0[r].z; acc[r].w += v0[r].w;
                if (two) {
                    acc[r].x += v1[r].x; acc[r].y += v1[r].y; acc[r].z += v1[r].z; acc[r].w += v1[r].w;
                }
            }
        }
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
            const int row = row0 + r_first + RPP * (rb + r);
            if (row >= M || col >= N) continue;
            float v[4] = {acc[r].x, acc[r].y, acc[r].z, acc[r].w};
            store4_c<OUT>(C, ldc, row, col, v, N, epi);
        }
    }
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
gemm_bf16_sm100_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmC,
                       const __grid_constant__ CUtensorMap tmBt,   // B, box of B_ROWS / 2 rows (narrow tail)
                       int M, int N, int K, void *C, int64_t ldc, int n_tma, int group_m, int wave_tiles,
                       int tail_first, int tail_parts,
                       DeviceStatus *status, uint64_t timeout_ns, uint32_t inject,
                       Epilogue epi, uint32_t layout,
                       float *sk_partials, unsigned long long *sk_counters, uint32_t sk_epoch,
                       const __grid_constant__ typename Cfg::PeerArg peers) {
    constexpr int CG = Cfg::CG;
    const bool a_mn = (layout & kLayoutAMajorM) != 0;   // A stored K x M
    const bool b_mn = (layout & kLayoutBMajorN) != 0;   // B stored K x N
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment of the shared-memory window offset (swizzle atoms).
    const uint32_t raw = smem_addr(smem_raw);
    uint8_t *smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
    const uint32_t base = smem_addr(smem);

    const uint32_t warp = threadIdx.x / 32;
    const uint32_t lane = threadIdx.x % 32;
    const uint32_t rank = (CG == 2) ? cluster_cta_rank() : 0u;
    // cluster split-K: this CTA's member index and the number of members
    const uint32_t kr = Cfg::SPLITK ? cluster_cta_rank() : 0u;
    const uint32_t ksplit = Cfg::SPLITK ? cluster_num_ctas() : 1u;
    const int cluster_ctas = Cfg::SPLITK ? static_cast<int>(ksplit) : CG;

    const uint32_t bar0 = base + Cfg::BAR_OFF;
    auto full_bar = [&](uint32_t s) { return bar0 + 8u * s; };
    auto empty_bar = [&](uint32_t s) { return bar0 + 8u * (Cfg::STAGES + s); };
    auto tfull_bar = [&](uint32_t b) { return bar0 + 8u * (2 * Cfg::STAGES + b); };
    auto tempty_bar = [&](uint32_t b) { return bar0 + 8u * (2 * Cfg::STAGES + 2 + b); };
    auto clc_bar = [&](uint32_t i) { return bar0 + 8u * (2 * Cfg::STAGES + 4 + i); };
    auto sched_full = [&](uint32_t i) { return bar0 + 8u * (2 * Cfg::STAGES + 6 + i); };
    auto sched_empty = [&](uint32_t i) { return bar0 + 8u * (2 * Cfg::STAGES + 8 + i); };
    // split-K: the other members' rings are free / their partials have arrived
    const uint32_t peer_free_bar = bar0 + 8u * (2 * Cfg::STAGES + 4 + (Cfg::CLC ? 6 : 0));
    const uint32_t rx_full_bar = peer_free_bar + 8u;
    const uint32_t tmem_slot = bar0 + 8u * Cfg::NUM_BARS;
    const uint32_t abort_slot = tmem_slot + 4u;
    const uint32_t tile_ids = tmem_slot + 8u;              // int32 [2]
    const uint32_t clc_resp = tmem_slot + 16u;             // 16-byte answers [2]
    volatile uint32_t *tmem_slot_ptr = reinterpret_cast<volatile uint32_t *>(smem + Cfg::BAR_OFF + 8 * Cfg::NUM_BARS);
    volatile uint32_t *abort_flag = tmem_slot_ptr + 1;
    volatile int32_t *tile_id_ptr = reinterpret_cast<volatile int32_t *>(tmem_slot_ptr + 2);
    volatile uint32_t *sk_last_flag = tmem_slot_ptr + 12;  // after the CLC answers

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 4 * CG);
        }
        if constexpr (Cfg::CLC) {
            for (int i = 0; i < 2; ++i) {
                mbar_init(clc_bar(i), 1);
                mbar_init(sched_full(i), 1);
                mbar_init(sched_empty(i), Cfg::SCHED_CONSUMERS);
            }
        }
        if constexpr (Cfg::SPLITK) {
            if (ksplit > 1) {
                mbar_init(peer_free_bar, ksplit - 1);            // one arrival per other member
                mbar_init(rx_full_bar, (ksplit - 1) * 128u);     // every epilogue thread of every other member
            }
        }
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_map(&tmA);
        tma_prefetch_map(&tmB);
        tma_prefetch_map(&tmC);
        if constexpr (Cfg::TAIL) tma_prefetch_map(&tmBt);
    }
    if (warp == 1) {
        tmem_alloc<CG>(tmem_slot, Cfg::TMEM_COLS);
        tmem_relinquish<CG>();
    }
    tc_fence_before_sync();
    __syncthreads();
    if constexpr (CG == 2 || Cfg::SPLITK) cluster_sync_all();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot_ptr;

    const int num_m = (M + Cfg::BM - 1) / Cfg::BM;
    const int num_n = (N + Cfg::BN - 1) / Cfg::BN;
    const int num_tiles = num_m * num_n;
    const int num_kb = (K + Cfg::BK - 1) / Cfg::BK;
    // Narrow tail (K-major B): units [0, tail_first) are whole tiles; tile
    // tail_first + i runs as unit tail_first + 2 i (columns [0, BN / 2)) and
    // unit tail_first + 2 i + 1 (columns [BN / 2, BN)).  Otherwise unit = tile.
    const int parts = (Cfg::TAIL && !b_mn && tail_parts == 2 && tail_first >= 0 && tail_first < num_tiles) ? 2 : 1;
    const int t_first = parts == 2 ? tail_first : num_tiles;
    const int num_units = t_first + (num_tiles - t_first) * parts;
    const int cluster_id = static_cast<int>(blockIdx.x) / cluster_ctas;
    const int num_clusters = static_cast<int>(gridDim.x) / cluster_ctas;
    // K blocks of every tile this CTA works on: all of them, or for split-K
    // this member's contiguous share
    const int kb_lo = Cfg::SPLITK ? static_cast<int>((static_cast<int64_t>(kr) * num_kb) / ksplit) : 0;
    const int kb_hi = Cfg::SPLITK ? static_cast<int>((static_cast<int64_t>(kr + 1) * num_kb) / ksplit) : num_kb;

    // The unit sequence every role of this CTA (and of its pair) walks.
    // Static: cluster_id, + num_clusters, ...  CLC: the first unit is the
    // cluster's own; the j-th later unit is read from ring slot j % 2, which
    // the scheduler warp fills, and the slot is handed back to the leader.
    auto next_tile = [&](int uid, uint32_t j, bool &ok) -> int {
        if constexpr (!Cfg::CLC) {
            (void)j;
            (void)ok;
            const int n = uid + num_clusters;
            return n < num_units ? n : -1;
        } else {
            (void)uid;
            const uint32_t slot = j & 1u;
            if (!mbar_wait(sched_full(slot), (j >> 1) & 1u, abort_flag, 3 * timeout_ns)) {
                ok = false;
                return -1;
            }
            const int n = tile_id_ptr[slot];
            if constexpr (CG == 1) mbar_arrive_local(sched_empty(slot));
            else mbar_arrive_cluster(map_to_cta(sched_empty(slot), 0));
            return n;
        }
    };

    // Work units: K blocks [kb0, kb1) of one tile (sub = -1), or of one half
    // of a narrow-tail tile (sub = 0, 1); uid is the unit's index in the
    // sequence the schedule hands out.  Static and CLC schedules: the units
    // from next_tile.  Stream-K with a data-parallel
    // head: with W >= 2 full waves of tiles, the first (W - 1) waves are whole
    // tiles dealt round robin (cluster c: c, c + G, ...); the (tile, K block)
    // iterations of the remaining tiles (one wave plus the partial one) are
    // cut into one contiguous range [it_begin, it_end) per cluster, one piece
    // per tile the range touches.  A cluster runs its split pieces (a range
    // boundary inside the tile: at most the first and the last) first, then
    // its data-parallel tiles, then its whole stream-K tiles: the tiles
    // shared with the neighbouring clusters complete early, so their fix-ups
    // overlap whole tiles instead of ending the launch.
    struct Unit {
        int tile, kb0, kb1, sub, uid;
    };
    auto unit_of = [&](int uid) -> Unit {
        if (!Cfg::TAIL || uid < t_first) return Unit{uid, kb_lo, kb_hi, -1, uid};
        const int r = uid - t_first;
        return Unit{t_first + r / parts, kb_lo, kb_hi, r % parts, uid};
    };
    const int64_t sk_waves = static_cast<int64_t>(num_tiles) / num_clusters;
    const int64_t dp_tiles = (Cfg::SK && sk_waves >= 2) ? (sk_waves - 1) * num_clusters : 0;
    const int dp_units = static_cast<int>(dp_tiles / num_clusters);     // data-parallel tiles per cluster
    const int64_t sk_base = dp_tiles * num_kb;                           // first stream-K iteration
    const int64_t sk_total = (static_cast<int64_t>(num_tiles) - dp_tiles) * num_kb;
    const int64_t it_begin = Cfg::SK ? sk_base + (static_cast<int64_t>(cluster_id) * sk_total) / num_clusters : 0;
    const int64_t it_end = Cfg::SK ? sk_base + (static_cast<int64_t>(cluster_id + 1) * sk_total) / num_clusters : 0;
    const int64_t sk_tile0 = it_begin / num_kb;
    const int sk_units = it_end > it_begin ? static_cast<int>((it_end - 1) / num_kb - sk_tile0 + 1) : 0;
    auto sk_range_unit = [&](int i) -> Unit {        // the i-th piece in range order
        Unit u;
        u.tile = static_cast<int>(sk_tile0 + i);
        const int64_t t0 = static_cast<int64_t>(u.tile) * num_kb;
        u.kb0 = static_cast<int>(max(it_begin - t0, int64_t(0)));
        u.kb1 = static_cast<int>(min(it_end - t0, static_cast<int64_t>(num_kb)));
        u.sub = -1;
        u.uid = u.tile;
        return u;
    };
    auto whole = [&](const Unit &u) { return u.kb0 == 0 && u.kb1 == num_kb; };
    const bool sk_split_first = Cfg::SK && sk_units > 0 && !whole(sk_range_unit(0));
    const bool sk_split_last = Cfg::SK && sk_units > 1 && !whole(sk_range_unit(sk_units - 1));
    auto sk_order = [&](int j) -> int {              // range position of the j-th piece run
        if (sk_split_last) {
            if (j == 0) return sk_units - 1;
            --j;
        }
        if (sk_split_first) {
            if (j == 0) return 0;
            --j;
        }
        return (sk_split_first ? 1 : 0) + j;
    };
    // the j-th unit this cluster runs: split stream-K pieces, data-parallel
    // tiles, whole stream-K tiles
    const int sk_split_units = (sk_split_last ? 1 : 0) + (sk_split_first ? 1 : 0);
    auto sk_unit = [&](int j) -> Unit {
        if (j < sk_split_units) return sk_range_unit(sk_order(j));
        if (j < sk_split_units + dp_units)
        {
            const int dt = cluster_id + (j - sk_split_units) * num_clusters;
            return Unit{dt, 0, num_kb, -1, dt};
        }
        return sk_range_unit(sk_order(j - dp_units));
    };
    auto first_unit = [&](Unit &u) -> bool {
        if constexpr (Cfg::SK) {
            if (sk_units + dp_units == 0) return false;
            u = sk_unit(0);
            return true;
        } else {
            u = unit_of(cluster_id);
            return cluster_id < num_units;
        }
    };
    // j counts the units this role has finished (the CLC ring position)
    auto next_unit = [&](Unit &u, uint32_t j, bool &ok) -> bool {
        if constexpr (Cfg::SK) {
            (void)ok;
            if (static_cast<int>(j) + 1 >= sk_units + dp_units) return false;
            u = sk_unit(static_cast<int>(j) + 1);
            return true;
        } else {
            const int n = next_tile(u.uid, j, ok);
            u = n >= 0 ? unit_of(n) : Unit{-1, kb_lo, kb_hi, -1, -1};
            return n >= 0;
        }
    };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer --
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            bool ok = true;
            const uint32_t leader_rank = 0;
            uint32_t fetched = 0;

            Unit u;
            for (bool more = first_unit(u); ok && more;) {
                const int tile = u.tile;
                int tm, tn;
                raster_tile(tile, num_m, num_n, group_m, tm, tn);
                const int a_row = tm * Cfg::BM + static_cast<int>(rank) * Cfg::BM_CTA;   // + c * BM_MMA
                // a narrow-tail half: B_ROWS / 2 rows per CTA, from tmBt
                const bool half = Cfg::TAIL && u.sub >= 0;
                const int b_row = half ? tn * Cfg::BN + u.sub * (Cfg::BN / 2) + static_cast<int>(rank) * (Cfg::B_ROWS / 2)
                                       : tn * Cfg::BN + static_cast<int>(rank) * Cfg::B_ROWS;
                const uint32_t tx = half ? static_cast<uint32_t>(CG * (Cfg::A_BYTES + Cfg::B_BYTES / 2))
                                         : static_cast<uint32_t>(Cfg::TX_BYTES);
                // Serpentine K: tiles of odd waves (tile / wave_tiles) walk K
                // backwards, so a new wave starts on the K slices of A and B
                // that the wave before it read last, which are still in L2.
                // The order is fixed per tile, so results stay deterministic.
                const bool rev = !Cfg::SK && !Cfg::SPLITK && wave_tiles > 0 && ((u.uid / wave_tiles) & 1) != 0;
                for (int kb = u.kb0; kb < u.kb1; ++kb) {
                    if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, 2 * timeout_ns)) {
                        record_timeout(status, abort_flag, abort_slot, cluster_ctas, kRoleProducer * 16 + kBarEmpty);
                        ok = false;
                        break;
                    }
                    const uint32_t a_dst = base + stage * Cfg::STAGE_BYTES;
                    const uint32_t b_dst = a_dst + Cfg::A_BYTES;
                    const int kx = (rev ? num_kb - 1 - kb : kb) * Cfg::BK;
                    if ((inject & kInjectDropFirstStage) && blockIdx.x == 0 && fetched == 0 && kb == u.kb0) {
                        // Failure-detection test: this stage's full barrier is
                        // never armed, so the MMA's bounded wait on it expires.
                        if (++stage == Cfg::STAGES) { stage = 0; phase ^= 1u; }
                        continue;
                    }
                    uint32_t bar;
                    if constexpr (CG == 1) {
                        bar = full_bar(stage);
                        mbar_arrive_expect_tx(bar, tx);
                    } else {
                        if (rank == leader_rank) mbar_arrive_expect_tx(full_bar(stage), tx);
                        bar = map_to_cta(full_bar(stage), leader_rank);
                    }
#pragma unroll
                    for (int c = 0; c < Cfg::CONSUMERS; ++c)
                        load_operand_tile<CG>(a_dst + c * Cfg::A_PART_BYTES, &tmA, bar, kx, a_row + c * Cfg::BM_MMA,
                                              Cfg::BM_CTA, a_mn);
                    if (half) load_operand_tile<CG>(b_dst, &tmBt, bar, kx, b_row, Cfg::B_ROWS / 2, false);
                    else load_operand_tile<CG>(b_dst, &tmB, bar, kx, b_row, Cfg::B_ROWS, b_mn);
                    if (++stage == Cfg::STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                more = next_unit(u, fetched++, ok);
                if (!ok) record_timeout(status, abort_flag, abort_slot, cluster_ctas, kRoleProducer * 16 + kBarSched);
            }
            // Tail: every stage handed out must be released by the MMA before
            // this CTA may exit (its empty barriers still receive arrivals).
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
        if (rank == 0 && lane == 0) {
            const uint32_t idesc_whole = idesc_bf16_f32(Cfg::BM_MMA, Cfg::BN, a_mn ? 1u : 0u, b_mn ? 1u : 0u);
            const uint32_t idesc_half = idesc_bf16_f32(Cfg::BM_MMA, Cfg::BN / 2, a_mn ? 1u : 0u, b_mn ? 1u : 0u);
            // Descriptors of stage 0, K step 0.  A stage, a consumer's A part
            // and a K step add their byte offset >> 4 to the start-address
            // field (bits 0-13), which cannot carry out: shared addresses
            // stay below 2^18.  One add per operand per MMA keeps the issue
            // loop as short as with compile-time layouts.
            const uint64_t a_desc0 = operand_desc(base, 0, a_mn);
            const uint64_t b_desc0 = operand_desc(base + Cfg::A_BYTES, 0, b_mn);
            const uint32_t a_kstep = (a_mn ? 2048u : 32u) >> 4;
            const uint32_t b_kstep = (b_mn ? 2048u : 32u) >> 4;
            uint32_t stage = 0, phase = 0;
            bool ok = true;
            int t = 0;
            Unit u;
            for (bool more = first_unit(u); ok && more; ++t) {
                const uint32_t buf = static_cast<uint32_t>(t) % Cfg::ACC_BUFS;
                const uint32_t acc_phase = (static_cast<uint32_t>(t) / Cfg::ACC_BUFS) & 1u;
                if (!mbar_wait(tempty_bar(buf), acc_phase ^ 1u, abort_flag, 3 * timeout_ns)) {
                    record_timeout(status, abort_flag, abort_slot, cluster_ctas, kRoleMma * 16 + kBarTmemEmpty);
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + buf * Cfg::CONSUMERS * Cfg::BN;
                const uint32_t idesc = (Cfg::TAIL && u.sub >= 0) ? idesc_half : idesc_whole;
                for (int kb = u.kb0; kb < u.kb1; ++kb) {
                    if (!mbar_wait(full_bar(stage), phase, abort_flag, timeout_ns)) {
                        record_timeout(status, abort_flag, abort_slot, cluster_ctas, kRoleMma * 16 + kBarFull);
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint64_t soff = (stage * Cfg::STAGE_BYTES) >> 4;
#pragma unroll
                    for (int kk = 0; kk < Cfg::BK / Cfg::UMMA_K; ++kk) {
                        const uint64_t bd = b_desc0 + soff + kk * b_kstep;
#pragma unroll
                        for (int c = 0; c < Cfg::CONSUMERS; ++c)   // both consumers read this B k-step
                            mma_bf16_ss<CG>(d_tmem + c * Cfg::BN,
                                            a_desc0 + soff + (c * Cfg::A_PART_BYTES >> 4) + kk * a_kstep, bd, idesc,
                                            (kb != u.kb0 || kk != 0) ? 1u : 0u);
                    }
                    mma_commit<CG>(empty_bar(stage), 0x3);
                    if (++stage == Cfg::STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                mma_commit<CG>(tfull_bar(buf), 0x3);
                more = next_unit(u, static_cast<uint32_t>(t), ok);
                if (!ok) record_timeout(status, abort_flag, abort_slot, cluster_ctas, kRoleMma * 16 + kBarSched);
            }
        }
        __syncwarp();
    } else if (Cfg::CLC && warp == 6) {
        // ------------------------------------------- CLC scheduler (leader) --
        if constexpr (Cfg::CLC) {
            if (rank == 0 && lane == 0) {
                for (uint32_t j = 0;; ++j) {
                    const uint32_t slot = j & 1u, ph = (j >> 1) & 1u;
                    if (!mbar_wait(sched_empty(slot), ph ^ 1u, abort_flag, 3 * timeout_ns)) {
                        record_timeout(status, abort_flag, abort_slot, cluster_ctas, kRoleScheduler * 16 + kBarSched);
                        break;
                    }
                    mbar_arrive_expect_tx(clc_bar(slot), 16);
                    clc_try_cancel(clc_resp + 16u * slot, clc_bar(slot));
                    if (!mbar_wait(clc_bar(slot), ph, abort_flag, 3 * timeout_ns)) {
                        record_timeout(status, abort_flag, abort_slot, cluster_ctas, kRoleScheduler * 16 + kBarClc);
                        break;
                    }
                    uint32_t first_x = 0;
                    const bool got = clc_query(clc_resp + 16u * slot, first_x);
                    fence_proxy_async_smem();   // the slot's answer is rewritten by a later request
                    const int next = got ? static_cast<int>(first_x) / CG : -1;
                    tile_id_ptr[slot] = next;
                    mbar_arrive_local(sched_full(slot));
                    if constexpr (CG == 2) {
                        store_cluster_s32(map_to_cta(tile_ids + 4u * slot, 1), next);
                        mbar_arrive_cluster(map_to_cta(sched_full(slot), 1));
                    }
                    if (next < 0) break;   // no cluster left: no further requests
                }
            }
        }
        __syncwarp();
    } else {
        // ----------------------------------------------------- epilogue --
        const uint32_t sub = warp & 3u;            // TMEM lanes [32*sub, 32*sub + 32)
        const uint32_t ew = warp - 2u;             // staging slot
        const bool fused = !epi.identity();
        const uint32_t stage_base = base + Cfg::STAGES * Cfg::STAGE_BYTES + ew * 2u * Cfg::EPI_BUF;
        const uint64_t c_policy = l2_policy_evict_first();
        uint32_t nstore = 0;
        int t = 0;
        Unit u;
        for (bool more = first_unit(u); more; ++t) {
            const int tile = u.tile;
            int tm, tn;
            raster_tile(tile, num_m, num_n, group_m, tm, tn);
            const uint32_t buf = static_cast<uint32_t>(t) % Cfg::ACC_BUFS;
            const uint32_t acc_phase = (static_cast<uint32_t>(t) / Cfg::ACC_BUFS) & 1u;
            // One lane waits; the result is broadcast so the warp stays
            // converged for the .sync.aligned TMEM loads below.
            uint32_t ready = 1;
            if (lane == 0 && !mbar_wait(tfull_bar(buf), acc_phase, abort_flag, 3 * timeout_ns)) {
                record_timeout(status, abort_flag, abort_slot, cluster_ctas, kRoleEpilogue * 16 + kBarTmemFull);
                ready = 0;
            }
            ready = __shfl_sync(0xffffffffu, ready, 0);
            if (!ready) break;
            tc_fence_after_sync();
            const int row_base = tm * Cfg::BM + static_cast<int>(rank) * Cfg::BM_CTA + static_cast<int>(sub) * 32;
            // a narrow-tail half: columns [sub BN / 2, (sub + 1) BN / 2) of the
            // tile, in accumulator columns [0, BN / 2)
            const bool half = Cfg::TAIL && u.sub >= 0;
            const int col0 = tn * Cfg::BN + (half ? u.sub * (Cfg::BN / 2) : 0);
            const uint32_t tbase0 = tmem_base + ((sub * 32u) << 16) + buf * Cfg::CONSUMERS * Cfg::BN;
            const int NQ = half ? Cfg::EPI_CHUNKS / 2 : Cfg::CONSUMERS * Cfg::EPI_CHUNKS;
            // chunk q: consumer q / EPI_CHUNKS (its own rows and accumulator),
            // columns (q % EPI_CHUNKS) * EPI_COLS of the tile
            auto chunk_taddr = [&](int q) -> uint32_t {
                const int cons = q / Cfg::EPI_CHUNKS, c = q - cons * Cfg::EPI_CHUNKS;
                return tbase0 + static_cast<uint32_t>(cons) * Cfg::BN + static_cast<uint32_t>(c * Cfg::EPI_COLS);
            };
            // This warp has read its whole slice of accumulator `buf`.
            auto release_tmem = [&]() {
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) {
                    if constexpr (CG == 1) mbar_arrive_local(tempty_bar(buf));
                    else mbar_arrive_cluster(map_to_cta(tempty_bar(buf), 0));
                }
            };
            // Write one chunk of C from registers (32 packed words: 32 fp32
            // or 64 bf16): the ragged end of each row by plain stores, the rest
            // through a swizzled staging buffer and a TMA store.
            auto store_chunk = [&](uint32_t (&packed)[32], int q) {
                const int cons = q / Cfg::EPI_CHUNKS, c = q - cons * Cfg::EPI_CHUNKS;
                const int row0 = row_base + cons * Cfg::BM_MMA;
                const int cstart = col0 + c * Cfg::EPI_COLS;
                if (cstart >= N) return;                    // chunk wholly right of C
                if (cstart + Cfg::EPI_COLS > n_tma) {
                    // Columns [n_tma, N) end C's rows inside a 16-byte granule:
                    // a TMA store writes whole granules, so these few elements
                    // (< 16 bytes per row) go out as plain predicated stores.
                    const int row = row0 + static_cast<int>(lane);
                    if (row < M) {
                        const int64_t roff = static_cast<int64_t>(row) * ldc * (Cfg::OUT == 0 ? 4 : 2);
                        auto tail = [&](void *dst) {
                            uint8_t *crow = static_cast<uint8_t *>(dst) + roff;
#pragma unroll
                            for (int w = 0; w < Cfg::EPI_COLS; ++w) {
                                const int col = cstart + w;
                                if (col >= n_tma && col < N) {
                                    if constexpr (Cfg::OUT == 0) {
                                        reinterpret_cast<uint32_t *>(crow)[col] = packed[w];
                                    } else {
                                        reinterpret_cast<uint16_t *>(crow)[col] =
                                            static_cast<uint16_t>(packed[w >> 1] >> (16 * (w & 1)));
                                    }
                                }
                            }
                        };
                        tail(C);
                        if constexpr (Cfg::PEERS)
                            for (int d = 0; d < peers.count; ++d) tail(peers.base[d]);
                    }
                    if (cstart >= n_tma) return;            // nothing left for the TMA store
                }
                const uint32_t sbuf = stage_base + (nstore & 1u) * Cfg::EPI_BUF;
                if (lane == 0) bulk_wait_group_read<1>();   // the store that used sbuf is done reading
                __syncwarp();
                // Row `lane` of the 32 x 128-byte box; 16-byte chunk j goes to
                // chunk slot j ^ (row % 8) -- the TMA 128-byte swizzle.
                const uint32_t row_addr = sbuf + lane * 128u;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    st_shared_v4(row_addr + ((static_cast<uint32_t>(j) ^ (lane & 7u)) << 4),
                                 packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    // C is written once and never read back by this kernel:
                    // its lines go first, so the A and B panels stay in L2
                    tma_store_2d_hint(&tmC, sbuf, cstart, row0, c_policy);
                    if constexpr (Cfg::PEERS)   // the same staged chunk to every other C
                        for (int d = 0; d < peers.count; ++d) tma_store_2d(&peers.map[d], sbuf, cstart, row0);
                    bulk_commit_group();
                }
                ++nstore;
            };
            bool split = false;   // stream-K: this unit is one piece of a split tile
            if constexpr (Cfg::SK) split = !(u.kb0 == 0 && u.kb1 == num_kb);
            if constexpr (Cfg::SPLITK) {
                // ---- cluster split-K: this member's accumulator holds the
                // fp32 partial over K blocks [u.kb0, u.kb1) (none: zeros).
                // Member j sums column slice j (SW columns) of the tile from
                // every member's partial, in member order, and writes it to
                // C.  Slice j of the others' partials crosses into member j's
                // operand ring, which its MMAs no longer read.
                const uint32_t S = ksplit;
                const int SW = Cfg::BN / static_cast<int>(S);      // a multiple of EPI_COLS (host)
                const bool has_k = u.kb1 > u.kb0;
                const uint32_t arow = sub * 32u + lane;            // accumulator row (TMEM lane)
                const uint32_t slot_bytes = 128u * static_cast<uint32_t>(SW) * 4u;
                const uint32_t epi_tid = threadIdx.x - 64u;
                auto load32 = [&](uint32_t col, uint32_t (&v)[32]) {
                    if (has_k) {
                        tmem_ld_32x32b_x32(tbase0 + col, v);
                        tmem_ld_wait();
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = 0u;
                    }
                };
                bool xok = true;
                if (S > 1) {
                    // this CTA's MMAs are done: its ring may take the others' partials
                    if (epi_tid == 0)
                        for (uint32_t j = 0; j < S; ++j)
                            if (j != kr) mbar_arrive_cluster(map_to_cta(peer_free_bar, j));
                    uint32_t fr = 1;
                    if (lane == 0 && !mbar_wait(peer_free_bar, 0, abort_flag, 3 * timeout_ns)) {
                        record_timeout(status, abort_flag, abort_slot, cluster_ctas, kRoleEpilogue * 16 + kBarPeerFree);
                        fr = 0;
                    }
                    xok = __shfl_sync(0xffffffffu, fr, 0) != 0;
                    __syncwarp();   // lane 0's acquire orders every lane's accesses that follow
                    if (xok) {
                        // slice j of this partial, row `arow`, to this member's slot
                        // at member j; 16-byte pieces swizzled by the row, so a
                        // warp's stores (and the reads back) are conflict-free
                        for (uint32_t j = 0; j < S; ++j) {
                            if (j == kr) continue;
                            const uint32_t slot = kr < j ? kr : kr - 1u;
                            const uint32_t dst_row =
                                map_to_cta(base + slot * slot_bytes + arow * static_cast<uint32_t>(SW) * 4u, j);
#pragma unroll 1
                            for (int c = 0; c < SW / 32; ++c) {
                                uint32_t v[32];
                                load32(j * static_cast<uint32_t>(SW) + static_cast<uint32_t>(c * 32), v);
#pragma unroll
                                for (int p = 0; p < 8; ++p) {
                                    const uint32_t piece = static_cast<uint32_t>(c * 8 + p) ^ (lane & 7u);
                                    store_cluster_v4(dst_row + (piece << 4), v[4 * p], v[4 * p + 1], v[4 * p + 2],
                                                     v[4 * p + 3]);
                                }
                            }
                            mbar_arrive_cluster(map_to_cta(rx_full_bar, j));   // release: the stores come first
                        }
                        uint32_t rf = 1;
                        if (lane == 0 && !mbar_wait(rx_full_bar, 0, abort_flag, 3 * timeout_ns)) {
                            record_timeout(status, abort_flag, abort_slot, cluster_ctas, kRoleEpilogue * 16 + kBarRxFull);
                            rf = 0;
                        }
                        xok = __shfl_sync(0xffffffffu, rf, 0) != 0;
                        __syncwarp();   // the other members' stores are visible to every lane
                    }
                }
                // 32 columns of slice kr (from slice column c * 32): the
                // members' partials added in member order
                auto slice_sum = [&](int c, uint32_t (&v)[32]) {
                    uint32_t own[32];
                    load32(kr * static_cast<uint32_t>(SW) + static_cast<uint32_t>(c * 32), own);
#pragma unroll 1
                    for (uint32_t m = 0; m < S; ++m) {
                        uint32_t x[32];
                        if (m == kr) {
#pragma unroll
                            for (int i = 0; i < 32; ++i) x[i] = own[i];
                        } else {
                            const uint32_t slot = m < kr ? m : m - 1u;
                            const uint32_t src_row = base + slot * slot_bytes + arow * static_cast<uint32_t>(SW) * 4u;
#pragma unroll
                            for (int p = 0; p < 8; ++p) {
                                const uint32_t piece = static_cast<uint32_t>(c * 8 + p) ^ (lane & 7u);
                                ld_shared_v4(src_row + (piece << 4), x[4 * p], x[4 * p + 1], x[4 * p + 2], x[4 * p + 3]);
                            }
                        }
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            v[i] = m == 0 ? x[i] : __float_as_uint(__uint_as_float(v[i]) + __uint_as_float(x[i]));
                    }
                };
                if (xok) {
                    const int erow = row_base + static_cast<int>(lane);
                    if constexpr (Cfg::OUT == 0) {
#pragma unroll 1
                        for (int c = 0; c < SW / 32; ++c) {
                            uint32_t v[32];
                            slice_sum(c, v);
                            const int q = static_cast<int>(kr) * SW / 32 + c;
                            if (fused) epilogue32_f32c(v, C, ldc, erow, col0 + q * 32, M, N, epi);
                            store_chunk(v, q);
                        }
                    } else {
#pragma unroll 1
                        for (int c = 0; c < SW / 32; c += 2) {
                            uint32_t v0[32], v1[32], packed[32];
                            slice_sum(c, v0);
                            slice_sum(c + 1, v1);
                            const int q = static_cast<int>(kr) * SW / 64 + c / 2;
                            if (fused) {
                                epilogue32_bf16c(v0, C, ldc, erow, col0 + q * 64, M, N, epi);
                                epilogue32_bf16c(v1, C, ldc, erow, col0 + q * 64 + 32, M, N, epi);
                            }
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                packed[i] = pack_bf16x2(__uint_as_float(v0[2 * i]), __uint_as_float(v0[2 * i + 1]));
                                packed[16 + i] = pack_bf16x2(__uint_as_float(v1[2 * i]), __uint_as_float(v1[2 * i + 1]));
                            }
                            store_chunk(packed, q);
                        }
                    }
                }
                release_tmem();
                if (!xok) break;
            } else if (split) {
              if constexpr (Cfg::SK) {
                // ---- stream-K: this unit is part of a tile split between
                // clusters.  Write this CTA's fp32 partial (row 32 sub + lane,
                // all BN columns) to its slot, count the arrival, and let the
                // last contributor sum every partial in contributor order.
                // (iterations counted from the first stream-K one)
                const int64_t G = num_clusters;
                auto owner = [&](int64_t it) { return ((it - sk_base + 1) * G + sk_total - 1) / sk_total - 1; };
                auto part = [&](int64_t cc) -> float * {
                    const int64_t first = (sk_base + (cc * sk_total) / G) / num_kb;   // cc's first stream-K tile
                    const int64_t slot = (cc * CG + rank) * 2 + (tile == first ? 0 : 1);
                    return sk_partials + slot * (128 * Cfg::BN);
                };
                const int64_t t0 = static_cast<int64_t>(tile) * num_kb;
                const int64_t c_lo = owner(t0), c_hi = owner(t0 + num_kb - 1);
                float *mine = part(cluster_id) + static_cast<int64_t>(sub * 32u + lane) * Cfg::BN;
#pragma unroll 1
                for (int c = 0; c < Cfg::BN / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tbase0 + static_cast<uint32_t>(c * 32), v);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        __stcg(reinterpret_cast<float4 *>(mine + c * 32 + 4 * j),
                               make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                           __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3])));
                }
                release_tmem();
                // The barrier orders the 128 threads' partial stores before
                // thread 0's gpu-scope fence, which (being cumulative) makes
                // them visible before its counter update.
                const uint32_t epi_tid = threadIdx.x - 64u;
                named_barrier_sync(1, 128);
                if (epi_tid == 0) {
                    __threadfence();
                    unsigned long long *ctr = sk_counters + static_cast<int64_t>(tile) * CG + rank;
                    const unsigned long long tag = static_cast<unsigned long long>(sk_epoch) << 32;
                    unsigned long long old = *reinterpret_cast<volatile unsigned long long *>(ctr), seen, want;
                    do {
                        seen = old;
                        want = ((seen & 0xFFFFFFFF00000000ull) == tag) ? seen + 1ull : (tag | 1ull);
                        old = atomicCAS(ctr, seen, want);
                    } while (old != seen);
                    *sk_last_flag =
                        ((want & 0xFFFFFFFFull) == static_cast<unsigned long long>(c_hi - c_lo + 1)) ? 1u : 0u;
                }
                named_barrier_sync(1, 128);
                if (*sk_last_flag) {
                    __threadfence();
                    sk_fixup<Cfg::OUT, Cfg::BN>(part, c_lo, c_hi,
                                                tm * Cfg::BM + static_cast<int>(rank) * Cfg::BM_CTA, col0, M, N, C, ldc,
                                                epi_tid, epi);
                    // all contributors have arrived: back to zero arrivals, so
                    // a replay of this launch (same epoch) starts clean
                    if (epi_tid == 0) sk_counters[static_cast<int64_t>(tile) * CG + rank] = static_cast<unsigned long long>(sk_epoch) << 32;
                }
                named_barrier_sync(1, 128);
              }
            } else if constexpr (Cfg::OUT == 0) {
                // fp32 C: one 32-column TMEM load per chunk, double-buffered in
                // registers so chunk q + 1's load is in flight while chunk q
                // is converted and stored
                auto finish = [&](uint32_t (&v)[32], int q) {
                    if (fused) {
                        const int cons = q / Cfg::EPI_CHUNKS, c = q - cons * Cfg::EPI_CHUNKS;
                        epilogue32_f32c(v, C, ldc, row_base + cons * Cfg::BM_MMA + static_cast<int>(lane),
                                        col0 + c * 32, M, N, epi);
                    }
                    store_chunk(v, q);
                };
                uint32_t ra[32], rb[32];
                tmem_ld_32x32b_x32(chunk_taddr(0), ra);
#pragma unroll 1
                for (int q = 0; q < NQ; q += 2) {
                    tmem_ld_wait();
                    if (q + 1 < NQ) tmem_ld_32x32b_x32(chunk_taddr(q + 1), rb);
                    else release_tmem();
                    finish(ra, q);
                    if (q + 1 < NQ) {
                        tmem_ld_wait();
                        if (q + 2 < NQ) tmem_ld_32x32b_x32(chunk_taddr(q + 2), ra);
                        else release_tmem();
                        finish(rb, q + 1);
                    }
                }
            } else {
#pragma unroll 1
                for (int q = 0; q < NQ; ++q) {
                    const int cons = q / Cfg::EPI_CHUNKS, c = q - cons * Cfg::EPI_CHUNKS;
                    const int erow = row_base + cons * Cfg::BM_MMA + static_cast<int>(lane);
                    uint32_t packed[32], v0[32], v1[32];
                    tmem_ld_32x32b_x32(chunk_taddr(q), v0);
                    tmem_ld_32x32b_x32(chunk_taddr(q) + 32, v1);
                    tmem_ld_wait();
                    if (q == NQ - 1) release_tmem();
                    if (fused) {
                        epilogue32_bf16c(v0, C, ldc, erow, col0 + c * 64, M, N, epi);
                        epilogue32_bf16c(v1, C, ldc, erow, col0 + c * 64 + 32, M, N, epi);
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        packed[i] = pack_bf16x2(__uint_as_float(v0[2 * i]), __uint_as_float(v0[2 * i + 1]));
                        packed[16 + i] = pack_bf16x2(__uint_as_float(v1[2 * i]), __uint_as_float(v1[2 * i + 1]));
                    }
                    store_chunk(packed, q);
                }
            }
            // next unit: stream-K computes it; otherwise one lane fetches the
            // next tile and the warp follows
            if constexpr (Cfg::SK) {
                bool ok = true;
                more = next_unit(u, static_cast<uint32_t>(t), ok);
            } else {
                int nt = -1;
                if (lane == 0) {
                    bool ok = true;
                    nt = next_tile(u.uid, static_cast<uint32_t>(t), ok);
                    if (!ok) record_timeout(status, abort_flag, abort_slot, cluster_ctas, kRoleEpilogue * 16 + kBarSched);
                }
                nt = __shfl_sync(0xffffffffu, nt, 0);
                u = nt >= 0 ? unit_of(nt) : Unit{-1, kb_lo, kb_hi, -1, -1};
                more = nt >= 0;
            }
        }
        if (lane == 0) bulk_wait_group<0>();
        __syncwarp();
    }

    // -------------------------------------------------------- teardown --
    tc_fence_before_sync();
    __syncthreads();
    if constexpr (CG == 2 || Cfg::SPLITK) cluster_sync_all();
    if (*abort_flag) {
        // A wait expired somewhere: give in-flight TMA copies and MMAs time
        // to land before the TMEM and shared memory are released.
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 200000ull) __nanosleep(1000);
    }
    __syncthreads();
    if constexpr (CG == 2 || Cfg::SPLITK) cluster_sync_all();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc<CG>(tmem_base, Cfg::TMEM_COLS);
    }
}

// C = 0 for K == 0 (the empty sum), one element per thread, grid-stride.
template <typename T>
__global__ void zero_fill_kernel(T *C, int64_t M, int64_t N, int64_t ldc) {
    const int64_t total = M * N;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = i / N;
        const int64_t c = i - r * N;
        C[r * ldc + c] = T(0);
    }
}

}  // namespace b200
