// Weight-streaming GEMM for a few rows: y[m, n] = sum_k x[m, k] W[n, k], then
// the GEMM epilogue, for M <= GEMV_MAX_M rows (a decode step's B sequences, the
// last-position logits). With so few rows each weight is used M times, so the
// operation is bound by reading W once from HBM; a 128-row tensor-core tile
// would leave most SMs idle (N / 256 tiles: 3 CTAs for N = 768).
//
// One warp per row n of W at a time, rows spread over every warp of the grid.
// Lane l reads 16 bytes of the row per step (256 bf16 or 128 fp32 elements per
// warp step) and the matching 16 bytes of each x row (x is small and stays in
// L1); the loop runs four steps deep so that each warp keeps 2 KB of W in
// flight. The M dot products are reduced across the warp with shuffles and
// lane m applies the epilogue to (m, n) exactly as the SIMT GEMM does
// (epilogue_scalar), so the numerics of every epilogue are those of the
// other engines in the same precision.
#include <algorithm>

#include "epilogue.cuh"

namespace gpt2 {

namespace {

constexpr int GV_THREADS = 256;

template <typename T>
struct GvVec;
template <>
struct GvVec<bf16> {
    static constexpr int N = 8;
    __device__ static void unpack(const uint4& q, float* f) {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 t = __bfloat1622float2(h[i]);
            f[2 * i] = t.x;
            f[2 * i + 1] = t.y;
        }
    }
};
template <>
struct GvVec<float> {
    static constexpr int N = 4;
    __device__ static void unpack(const uint4& q, float* f) {
        f[0] = __uint_as_float(q.x);
        f[1] = __uint_as_float(q.y);
        f[2] = __uint_as_float(q.z);
        f[3] = __uint_as_float(q.w);
    }
};

template <typename T, int MM>
__global__ void __launch_bounds__(GV_THREADS) gemv_kernel(const T* __restrict__ x, const T* __restrict__ W, int N,
                                                          int K, Epilogue ep) {
    constexpr int VE = GvVec<T>::N;
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (GV_THREADS / 32);
    const int K16 = K / VE;   // 16-byte pieces per row
    for (int n = blockIdx.x * (GV_THREADS / 32) + (threadIdx.x >> 5); n < N; n += warps) {
        const uint4* wr = reinterpret_cast<const uint4*>(W + (long long)n * K);
        float acc[MM];
#pragma unroll
        for (int m = 0; m < MM; ++m) acc[m] = 0.f;
#pragma unroll 4
        for (int j = lane; j < K16; j += 32) {
            float w[VE];
            GvVec<T>::unpack(__ldg(wr + j), w);
#pragma unroll
            for (int m = 0; m < MM; ++m) {
                float a[VE];
                GvVec<T>::unpack(__ldg(reinterpret_cast<const uint4*>(x + (long long)m * K) + j), a);
#pragma unroll
                for (int e = 0; e < VE; ++e) acc[m] = fmaf(a[e], w[e], acc[m]);
            }
        }
#pragma unroll
        for (int m = 0; m < MM; ++m) acc[m] = warp_sum(acc[m]);
        // lane m applies the epilogue to output (m, n)
#pragma unroll
        for (int m = 0; m < MM; ++m)
            if (lane == m) epilogue_scalar<T>(ep, m, n, 1, &acc[m]);
    }
}

template <typename T, int MM>
void launch_mm(const Ctx& ctx, const T* x, const T* W, int N, int K, const Epilogue& ep) {
    const int warps_needed = N;
    const int blocks = std::min(ceil_div(warps_needed, GV_THREADS / 32), 8 * (ctx.num_sms > 0 ? ctx.num_sms : 148));
    gemv_kernel<T, MM><<<blocks, GV_THREADS, 0, ctx.stream>>>(x, W, N, K, ep);
}

}  // namespace

bool gemv_supported(size_t elem_size, int M, int K) {
    return M >= 1 && M <= GEMV_MAX_M && K >= 1 && (K * elem_size) % 16 == 0;
}

template <typename T>
void launch_gemv(const Ctx& ctx, const T* x, const T* W, int M, int N, int K, const Epilogue& ep) {
    switch (M) {
    case 1: launch_mm<T, 1>(ctx, x, W, N, K, ep); break;
    case 2: launch_mm<T, 2>(ctx, x, W, N, K, ep); break;
    case 3: launch_mm<T, 3>(ctx, x, W, N, K, ep); break;
    default: launch_mm<T, 4>(ctx, x, W, N, K, ep); break;
    }
    ++*ctx.launches;
}

template void launch_gemv<float>(const Ctx&, const float*, const float*, int, int, int, const Epilogue&);
template void launch_gemv<bf16>(const Ctx&, const bf16*, const bf16*, int, int, int, const Epilogue&);

}  // namespace gpt2
