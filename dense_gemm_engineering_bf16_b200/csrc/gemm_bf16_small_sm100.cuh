// Latency path for tiny bf16 GEMMs on sm_100a: C = act(alpha A.B + beta C + bias).
//
// For a product of a few MFLOP the tcgen05 kernels spend most of their time
// before the first MMA and after the last one: tensor memory is allocated
// and freed, barriers are set up, and a pipeline of TMA stages fills and
// drains.  Here each warp computes a 16 x 16 block of C with the warp-level
// tensor-core instruction mma.sync m16n8k16 (bf16 inputs, fp32
// accumulation): no tensor memory, no mbarriers, one ordinary launch.  It is
// the latency entry of the pages' autotune search space ("GPU 执行模型",
// section "编译与 autotune": the kernel choice per shape), used only below a
// work bound measured on the GPU; every larger product takes the tcgen05
// kernels.
//
// CTA: 4 warps, a 32 x 32 tile of C; warp w takes rows 16 (w / 2) and
// columns 16 (w % 2) of it, as two m16n8 accumulators.  K-major operands
// (A as M x K, B as N x K) are staged in shared memory with cp.async, 128 K
// at a time, two chunks in flight, so a K of up to 128 costs one round trip
// to memory; 16-byte copies zero-fill past M, N and K.  MN-major operands
// (forced, or through gemm_bf16_ex / gemm_bf16_fused) are read straight from
// global memory, two elements at a time.  Fragment layout of
// mma.sync.m16n8k16 (PTX ISA, "Matrix fragments for mma.m16n8k16"), with
// g = lane / 4 and t = lane % 4:
//   A (16 x 16, row):  a0 = A[g][2t, 2t+1]      a1 = A[g+8][2t, 2t+1]
//                      a2 = A[g][2t+8, 2t+9]    a3 = A[g+8][2t+8, 2t+9]
//   B (16 x 8, col):   b0 = B[2t, 2t+1][g]      b1 = B[2t+8, 2t+9][g]
//   C (16 x 8):        c0, c1 = C[g][2t, 2t+1]  c2, c3 = C[g+8][2t, 2t+1]
// (two bf16 per 32-bit register, the lower K index in the low half).
// Elements outside M, N or K read as zero; stores are bounded by M and N.
#pragma once
#include <cuda_bf16.h>

#include <cstdint>

#include "epilogue.cuh"
#include "gemm_bf16_sm100.cuh"

namespace b200 {

// Two consecutive K elements (k, k + 1) of row `row` of an operand, packed
// as bf16x2; zeros past `rows` or K.  K-major (row-major [rows][ld]): one
// 32-bit load when both are in range (k is even and ld a multiple of 8, so
// the address is 4-byte aligned).  MN-major ([K][ld], the row index
// fastest): two 16-bit loads.
__device__ __forceinline__ uint32_t small_pair(const uint16_t *P, int64_t ld, bool mn, int row, int rows, int k,
                                               int K) {
    if (row >= rows || k >= K) return 0u;
    if (!mn) {
        const uint16_t *p = P + static_cast<int64_t>(row) * ld + k;
        if (k + 1 < K) return *reinterpret_cast<const uint32_t *>(p);
        return static_cast<uint32_t>(p[0]);
    }
    const uint32_t lo = P[static_cast<int64_t>(k) * ld + row];
    const uint32_t hi = k + 1 < K ? P[static_cast<int64_t>(k + 1) * ld + row] : 0u;
    return lo | (hi << 16);
}

__device__ __forceinline__ void mma_m16n8k16_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                                  uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

constexpr int kSmallKC = 128;                 // K per staged chunk
constexpr int kSmallRow = kSmallKC + 8;        // staged row pitch (elements): 272 bytes, conflict-free reads

// 16-byte global -> shared copy; `bytes` (0..16) are read, the rest zero-filled.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src, uint32_t bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int OUT>
__device__ __forceinline__ void small_store(void *C, int64_t ldc, int M, int N, int m0, int n0, int g, int t,
                                            const float (&acc)[2][4], const Epilogue &epi) {
#pragma unroll
    for (int f = 0; f < 2; ++f) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int row = m0 + g + (r >= 2 ? 8 : 0);
            const int col = n0 + 8 * f + 2 * t + (r & 1);
            if (row >= M || col >= N) continue;
            const int64_t i = static_cast<int64_t>(row) * ldc + col;
            const float b = epi.bias ? epi.bias[col] : 0.0f;
            if constexpr (OUT == 0) {
                float *c = static_cast<float *>(C);
                c[i] = finish(acc[f][r], epi.beta != 0.0f ? c[i] : 0.0f, b, epi);
            } else {
                __nv_bfloat16 *c = static_cast<__nv_bfloat16 *>(C);
                c[i] = __float2bfloat16_rn(finish(acc[f][r], epi.beta != 0.0f ? __bfloat162float(c[i]) : 0.0f, b,
                                                  epi));
            }
        }
    }
}

// K-major A and B: 32 rows of each, 128 K per chunk, staged in shared memory.
template <int OUT>
__global__ void __launch_bounds__(128)
gemm_bf16_small_kmajor_kernel(const uint16_t *__restrict__ A, const uint16_t *__restrict__ B, void *C, int M,
                              int N, int K, int64_t lda, int64_t ldb, int64_t ldc, Epilogue epi) {
    __shared__ __align__(16) uint16_t sA[2][32][kSmallRow];
    __shared__ __align__(16) uint16_t sB[2][32][kSmallRow];
    const int tid = static_cast<int>(threadIdx.x);
    const int warp = tid / 32, lane = tid % 32;
    const int g = lane / 4, t = lane % 4;
    const int mb = static_cast<int>(blockIdx.y) * 32, nb = static_cast<int>(blockIdx.x) * 32;
    const int wr = (warp / 2) * 16, wc = (warp % 2) * 16;
    // chunk c into buffer c % 2: per operand 32 rows x 16 segments of 8 K,
    // four segments per thread
    auto load_chunk = [&](int c) {
        const int buf = c & 1, k0 = c * kSmallKC;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int seg = tid + 128 * i;
            const int r = seg / 16, k = k0 + (seg % 16) * 8;
            const int kb = K - k < 8 ? (K - k) * 2 : 16;            // bytes of this segment inside K
            const int ar = mb + r, br = nb + r;
            const uint32_t ab = (ar < M && k < K) ? static_cast<uint32_t>(kb) : 0u;
            const uint32_t bb = (br < N && k < K) ? static_cast<uint32_t>(kb) : 0u;
            cp_async_16(static_cast<uint32_t>(__cvta_generic_to_shared(&sA[buf][r][(seg % 16) * 8])),
                        ab ? static_cast<const void *>(A + static_cast<int64_t>(ar) * lda + k) : A, ab);
            cp_async_16(static_cast<uint32_t>(__cvta_generic_to_shared(&sB[buf][r][(seg % 16) * 8])),
                        bb ? static_cast<const void *>(B + static_cast<int64_t>(br) * ldb + k) : B, bb);
        }
        cp_async_commit();
    };
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    const int chunks = (K + kSmallKC - 1) / kSmallKC;
    load_chunk(0);
    for (int c = 0; c < chunks; ++c) {
        if (c + 1 < chunks) {
            load_chunk(c + 1);            // its buffer was last read in chunk c - 1, before the barrier below
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const int buf = c & 1;
#pragma unroll
        for (int kk = 0; kk < kSmallKC; kk += 16) {
            uint32_t a[4];
            a[0] = *reinterpret_cast<const uint32_t *>(&sA[buf][wr + g][kk + 2 * t]);
            a[1] = *reinterpret_cast<const uint32_t *>(&sA[buf][wr + g + 8][kk + 2 * t]);
            a[2] = *reinterpret_cast<const uint32_t *>(&sA[buf][wr + g][kk + 2 * t + 8]);
            a[3] = *reinterpret_cast<const uint32_t *>(&sA[buf][wr + g + 8][kk + 2 * t + 8]);
#pragma unroll
            for (int f = 0; f < 2; ++f) {
                const uint32_t b0 = *reinterpret_cast<const uint32_t *>(&sB[buf][wc + 8 * f + g][kk + 2 * t]);
                const uint32_t b1 = *reinterpret_cast<const uint32_t *>(&sB[buf][wc + 8 * f + g][kk + 2 * t + 8]);
                mma_m16n8k16_bf16(acc[f], a, b0, b1);
            }
        }
        __syncthreads();                  // every warp is done with this buffer
    }
    small_store<OUT>(C, ldc, M, N, mb + wr, nb + wc, g, t, acc, epi);
}

// Any layout: fragments read straight from global memory.
template <int OUT>
__global__ void __launch_bounds__(128)
gemm_bf16_small_kernel(const uint16_t *__restrict__ A, const uint16_t *__restrict__ B, void *C, int M, int N,
                       int K, int64_t lda, int64_t ldb, int64_t ldc, uint32_t layout, Epilogue epi) {
    const bool a_mn = (layout & kLayoutAMajorM) != 0;   // A stored K x M
    const bool b_mn = (layout & kLayoutBMajorN) != 0;   // B stored K x N
    const int warp = static_cast<int>(threadIdx.x) / 32;
    const int lane = static_cast<int>(threadIdx.x) % 32;
    const int g = lane / 4, t = lane % 4;
    const int m0 = static_cast<int>(blockIdx.y) * 32 + (warp / 2) * 16;
    const int n0 = static_cast<int>(blockIdx.x) * 32 + (warp % 2) * 16;
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 4
    for (int k0 = 0; k0 < K; k0 += 16) {
        uint32_t a[4];
        a[0] = small_pair(A, lda, a_mn, m0 + g, M, k0 + 2 * t, K);
        a[1] = small_pair(A, lda, a_mn, m0 + g + 8, M, k0 + 2 * t, K);
        a[2] = small_pair(A, lda, a_mn, m0 + g, M, k0 + 2 * t + 8, K);
        a[3] = small_pair(A, lda, a_mn, m0 + g + 8, M, k0 + 2 * t + 8, K);
#pragma unroll
        for (int f = 0; f < 2; ++f) {
            const int n = n0 + 8 * f + g;
            const uint32_t b0 = small_pair(B, ldb, b_mn, n, N, k0 + 2 * t, K);
            const uint32_t b1 = small_pair(B, ldb, b_mn, n, N, k0 + 2 * t + 8, K);
            mma_m16n8k16_bf16(acc[f], a, b0, b1);
        }
    }
    small_store<OUT>(C, ldc, M, N, m0, n0, g, t, acc, epi);
}

}  // namespace b200
