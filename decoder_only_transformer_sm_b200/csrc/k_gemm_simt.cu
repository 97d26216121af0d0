// SIMT GEMM with fp32 FMA accumulation: the fp32-mode contraction (no TF32, so
// that fp32 results stay within 1e-4 of a float64 reference) for every layout.
#include "epilogue.cuh"

namespace gpt2 {

namespace {

constexpr int SB_M = 64, SB_N = 64, SB_K = 16, S_THREADS = 256;

template <typename T>
__global__ void __launch_bounds__(S_THREADS) gemm_simt_kernel(int layout, const T* __restrict__ A,
                                                              const T* __restrict__ B, int M, int N, int K,
                                                              Epilogue ep) {
    __shared__ float As[SB_K][SB_M + 4];
    __shared__ float Bs[SB_K][SB_N + 4];
    const int tid = threadIdx.x;
    const int m0 = blockIdx.y * SB_M, n0 = blockIdx.x * SB_N;
    const int tr = tid / 16, tc = tid % 16;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    for (int k0 = 0; k0 < K; k0 += SB_K) {
        // A(m, k): row-major [M,K] (NT, NN) or [K,M] (TN)
        for (int i = tid; i < SB_M * SB_K; i += S_THREADS) {
            int mm, kk;
            if (layout == GEMM_TN) { mm = i % SB_M; kk = i / SB_M; }
            else { kk = i % SB_K; mm = i / SB_K; }
            const int gm = m0 + mm, gk = k0 + kk;
            float v = 0.f;
            if (gm < M && gk < K)
                v = to_f(layout == GEMM_TN ? A[(long long)gk * M + gm] : A[(long long)gm * K + gk]);
            As[kk][mm] = v;
        }
        // B(n, k): row-major [N,K] (NT) or [K,N] (NN, TN)
        for (int i = tid; i < SB_N * SB_K; i += S_THREADS) {
            int nn, kk;
            if (layout == GEMM_NT) { kk = i % SB_K; nn = i / SB_K; }
            else { nn = i % SB_N; kk = i / SB_N; }
            const int gn = n0 + nn, gk = k0 + kk;
            float v = 0.f;
            if (gn < N && gk < K)
                v = to_f(layout == GEMM_NT ? B[(long long)gn * K + gk] : B[(long long)gk * N + gn]);
            Bs[kk][nn] = v;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < SB_K; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][tr * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tc * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int row = m0 + tr * 4 + i;
        const int col = n0 + tc * 4;
        if (row < M && col < N) epilogue_run<T, 4>(ep, row, col, N, acc[i]);
    }
}

}  // namespace

template <typename T>
void launch_gemm_simt(const Ctx& ctx, GemmLayout layout, const T* A, const T* B, int M, int N, int K,
                      const Epilogue& ep) {
    dim3 grid(ceil_div(N, SB_N), ceil_div(M, SB_M));
    gemm_simt_kernel<T><<<grid, S_THREADS, 0, ctx.stream>>>((int)layout, A, B, M, N, K, ep);
    ++*ctx.launches;
}

template void launch_gemm_simt<float>(const Ctx&, GemmLayout, const float*, const float*, int, int, int,
                                      const Epilogue&);
template void launch_gemm_simt<bf16>(const Ctx&, GemmLayout, const bf16*, const bf16*, int, int, int,
                                     const Epilogue&);

}  // namespace gpt2
