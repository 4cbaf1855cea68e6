// Fused GEMM write-back: C = act(alpha * acc + beta * C_old + bias[col]),
// applied to the fp32 accumulator in registers before the single rounding to
// the output type, so the intermediate never makes a round trip through HBM
// ("GPU 执行模型", section "Fusion 的收益与上限": about two intermediate-sized
// transfers saved per fused pointwise step).
#pragma once

#include <cstdint>

namespace b200 {

enum : uint32_t { kActNone = 0, kActRelu = 1, kActGelu = 2, kActGeluTanh = 3, kActCount = 4 };

struct Epilogue {
    float alpha;
    float beta;          // C_old is read only when beta != 0
    const float *bias;   // N fp32 values, 16-byte aligned, or nullptr
    uint32_t act;        // kAct*

    __host__ __device__ bool identity() const {
        return alpha == 1.0f && beta == 0.0f && bias == nullptr && act == kActNone;
    }
};

__host__ __device__ inline Epilogue plain_epilogue() { return Epilogue{1.0f, 0.0f, nullptr, kActNone}; }

// The hardware tanh approximation (PTX tanh.approx.f32, one MUFU op).
__device__ __forceinline__ float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float activate(float x, uint32_t act) {
    if (act == kActRelu) return x < 0.0f ? 0.0f : x;                       // NaN passes through
    if (act == kActGelu) return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f));   // x Phi(x)
    if (act == kActGeluTanh) {
        // 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))), the tanh form of GELU
        const float u = 0.79788456080286536f * fmaf(0.044715f * x, x * x, x);
        return 0.5f * x * (1.0f + tanh_approx(u));
    }
    return x;
}

// One element: the order is alpha * acc (+ beta * old) (+ bias), then act.
// The bias is added only when present, so a -0 product stays -0.
__device__ __forceinline__ float finish(float acc, float old, float bias, const Epilogue &e) {
    float x = e.beta != 0.0f ? fmaf(e.alpha, acc, e.beta * old) : e.alpha * acc;
    if (e.bias) x += bias;
    return activate(x, e.act);
}

// bias[col0 + j] for j < 32 (0 past N or without a bias); all lanes of a warp
// read the same addresses, so each load is one broadcast.
__device__ __forceinline__ void load_bias32(float (&b)[32], const float *bias, int col0, int N) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const int col = col0 + 4 * q;
        if (bias && col + 4 <= N) {
            const float4 x = __ldg(reinterpret_cast<const float4 *>(bias + col));
            b[4 * q] = x.x; b[4 * q + 1] = x.y; b[4 * q + 2] = x.z; b[4 * q + 3] = x.w;
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) b[4 * q + e] = (bias && col + e < N) ? __ldg(bias + col + e) : 0.0f;
        }
    }
}

// 32 fp32 accumulators (as bits) of row `row`, columns col0.., whose C is
// fp32: v <- finish(v, C_old, bias).  C is read only inside M x N.
__device__ __forceinline__ void epilogue32_f32c(uint32_t (&v)[32], const void *C, int64_t ldc, int row, int col0,
                                                int M, int N, const Epilogue &e) {
    const float *crow = static_cast<const float *>(C) + static_cast<int64_t>(row) * ldc;
    float b[32];
    load_bias32(b, e.bias, col0, N);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        float old[4] = {0.f, 0.f, 0.f, 0.f};
        const int col = col0 + 4 * q;
        if (e.beta != 0.0f && row < M) {
            if (col + 4 <= N) {
                const float4 x = *reinterpret_cast<const float4 *>(crow + col);
                old[0] = x.x; old[1] = x.y; old[2] = x.z; old[3] = x.w;
            } else {
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    if (col + k < N) old[k] = crow[col + k];
            }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k)
            v[4 * q + k] = __float_as_uint(finish(__uint_as_float(v[4 * q + k]), old[k], b[4 * q + k], e));
    }
}

// The same for 32 fp32 accumulators whose C elements are bf16.
__device__ __forceinline__ void epilogue32_bf16c(uint32_t (&v)[32], const void *C, int64_t ldc, int row, int col0,
                                                 int M, int N, const Epilogue &e) {
    const uint16_t *crow = static_cast<const uint16_t *>(C) + static_cast<int64_t>(row) * ldc;
    float b[32];
    load_bias32(b, e.bias, col0, N);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t w[4] = {0u, 0u, 0u, 0u};
        const int col = col0 + 8 * q;
        if (e.beta != 0.0f && row < M) {
            if (col + 8 <= N) {
                const uint4 x = *reinterpret_cast<const uint4 *>(crow + col);
                w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    if (col + k < N) w[k >> 1] |= static_cast<uint32_t>(crow[col + k]) << (16 * (k & 1));
            }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float old = __uint_as_float((w[k >> 1] >> (16 * (k & 1))) << 16);   // bf16 -> f32
            v[8 * q + k] = __float_as_uint(finish(__uint_as_float(v[8 * q + k]), old, b[8 * q + k], e));
        }
    }
}

// C = act(beta * C + bias) over M x N when K = 0 (the empty product); C is
// read only when beta != 0.  Block-strided over rows, threads over 16-byte
// vectors of a row (every row starts 16-byte aligned: C and ldc * sizeof(T)
// are), so the pass streams C at close to HBM bandwidth; run on its own
// after a plain GEMM it is also the unfused form of the fused epilogue.
template <typename T>
__global__ void epilogue_only_kernel(T *C, int64_t M, int64_t N, int64_t ldc, Epilogue e) {
    constexpr int V = 16 / sizeof(T);
    const int64_t nvec = N / V;
    for (int64_t r = blockIdx.x; r < M; r += gridDim.x) {
        T *row = C + r * ldc;
        for (int64_t v = threadIdx.x; v < nvec; v += blockDim.x) {
            const int64_t c0 = v * V;
            uint4 w = make_uint4(0u, 0u, 0u, 0u);
            if (e.beta != 0.0f) w = *reinterpret_cast<const uint4 *>(row + c0);
            const T *x = reinterpret_cast<const T *>(&w);
            alignas(16) T y[V];
#pragma unroll
            for (int k = 0; k < V; ++k) {
                const float old = e.beta != 0.0f ? static_cast<float>(x[k]) : 0.0f;
                const float b = e.bias ? __ldg(e.bias + c0 + k) : 0.0f;
                y[k] = static_cast<T>(finish(0.0f, old, b, e));
            }
            *reinterpret_cast<uint4 *>(row + c0) = *reinterpret_cast<const uint4 *>(y);
        }
        for (int64_t c = nvec * V + threadIdx.x; c < N; c += blockDim.x) {   // ragged end of the row
            const float old = e.beta != 0.0f ? static_cast<float>(row[c]) : 0.0f;
            const float b = e.bias ? e.bias[c] : 0.0f;
            row[c] = static_cast<T>(finish(0.0f, old, b, e));
        }
    }
}

}  // namespace b200
