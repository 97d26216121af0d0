// Weight-streaming GEMM for a few rows: y[m, n] = sum_k x[m, k] W[n, k], then
// the GEMM epilogue, for M <= GEMV_MAX_M rows (a decode step's B sequences, the
// last-position logits). With so few rows each weight is used M times, so the
// operation is bound by reading W once from HBM; a 128-row tensor-core tile
// would leave most SMs idle (N / 256 tiles: 3 CTAs for N = 768).
//
// Work split: W's rows in groups of RG consecutive rows, one group per warp at
// a time, groups spread over every warp of the grid (RG picked so that there
// are a few groups per SM). Lane l reads 16 bytes of each of the RG rows per
// step (256 bf16 or 128 fp32 elements per warp step), up to U steps ahead,
// so each lane keeps RG * U 16-byte loads in flight; the matching 16 bytes
// of each x row come from L1 or shared memory. The M * RG dot products are
// reduced across the warp with shuffles and lane r*M + m applies the epilogue
// to (m, n0 + r) exactly as the SIMT GEMM does (epilogue_scalar), so every
// epilogue has the numerics of the other engines in the same precision.
//
// Fused LayerNorm (ln.x set): x is not read from memory but computed by each
// block into shared memory as LN(ln.x[m, :]) with (ln.w, ln.b), one warp per
// row, in launch_layernorm_fwd's arithmetic and order ("GPT-2 from Scratch",
// "The Block: pre-LN and residuals": eps 1e-5, biased variance), rounded to
// the operand type.
//
// Launch: programmatic dependent launch when ctx.pdl. Before griddep_wait a
// warp loads the first U steps of its first row group into registers and
// starts the fetch of its other row groups into L2 (a bulk prefetch each): the
// weights do not depend on the previous kernel, so their fetch overlaps its
// tail. If ep.out_row_dev is set, the output base moves on by
// *out_row_dev rows of out_row_bytes, read on the device (the key/value cache
// row of a replayed decode step).
#include <algorithm>

#include "epilogue.cuh"

namespace gpt2 {

namespace {

constexpr int GV_WARPS = 4;
constexpr int GV_THREADS = 32 * GV_WARPS;

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

__device__ __forceinline__ void prefetch_l2_bulk(const void* p, unsigned bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ void prefetch_l1(const void* p) { asm volatile("prefetch.global.L1 [%0];" ::"l"(p)); }

// y = LN(x) over C columns by one warp (lane l: float4 chunks l, l + 32, ...).
template <typename T>
__device__ __forceinline__ void ln_row(const float* __restrict__ x, const float* __restrict__ w,
                                       const float* __restrict__ b, int C, T* __restrict__ y, int lane) {
    float s = 0.f;
    for (int c = lane * 4; c < C; c += 128) {
        float v[4];
        load4(x + c, v);
#pragma unroll
        for (int j = 0; j < 4; ++j) s += v[j];
    }
    const float mu = warp_sum(s) / C;
    float ss = 0.f;
    for (int c = lane * 4; c < C; c += 128) {
        float v[4];
        load4(x + c, v);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float d = v[j] - mu;
            ss += d * d;
        }
    }
    const float rs = rsqrtf(warp_sum(ss) / C + 1e-5f);
    for (int c = lane * 4; c < C; c += 128) {
        float v[4], ww[4], bb[4], o[4];
        load4(x + c, v);
        load4(w + c, ww);
        load4(b + c, bb);
#pragma unroll
        for (int j = 0; j < 4; ++j) o[j] = (v[j] - mu) * rs * ww[j] + bb[j];
        store4(y + c, o);
    }
}

template <typename T, int RG, int U>
__device__ __forceinline__ void load_w(const uint4* const (&wr)[RG], int j0, int K16, uint4 (&wq)[RG][U]) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int j = j0 + 32 * u;
#pragma unroll
        for (int r = 0; r < RG; ++r) wq[r][u] = j < K16 ? __ldg(wr[r] + j) : make_uint4(0, 0, 0, 0);
    }
}

template <typename T, int MM, int RG, int U, bool LN>
__global__ void __launch_bounds__(GV_THREADS) gemv_kernel(const T* __restrict__ x, const T* __restrict__ W, int N,
                                                          int K, Epilogue ep, LnIn ln) {
    extern __shared__ __align__(16) unsigned char gv_smem[];
    T* xs = reinterpret_cast<T*>(gv_smem);   // LN: MM rows of K
    constexpr int VE = GvVec<T>::N;
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const int warps = gridDim.x * GV_WARPS;
    const int K16 = K / VE;   // 16-byte pieces per row
    const int groups = (N + RG - 1) / RG;
    const int g0 = blockIdx.x * GV_WARPS + wib;
    griddep_launch();
    // Work that does not depend on the previous kernel: the fetch of this warp's
    // W rows into L2, and the first U steps of its first row group into registers.
    if (lane == 0 && (reinterpret_cast<uintptr_t>(W) & 15) == 0) {
        for (int g = g0 + warps; g < groups; g += warps) {
            const int n0 = g * RG;
            prefetch_l2_bulk(W + (long long)n0 * K, (unsigned)(min(RG, N - n0) * K * (int)sizeof(T)));
        }
    }
    uint4 wq[RG][U];
    const uint4* wr[RG];
    if (g0 < groups) {
#pragma unroll
        for (int r = 0; r < RG; ++r)
            wr[r] = reinterpret_cast<const uint4*>(W + (long long)min(g0 * RG + r, N - 1) * K);   // past N: unused
        load_w<T, RG, U>(wr, lane, K16, wq);
        if (ep.bias && lane == 0) prefetch_l1(ep.bias + g0 * RG);   // the first group's bias
    }
    if (LN) {   // the LayerNorm parameters, one 128-byte line per lane step
        for (int c = threadIdx.x * 32; c < K; c += GV_THREADS * 32) {
            prefetch_l1(ln.w + c);
            prefetch_l1(ln.b + c);
        }
    }
    griddep_wait();
    if (ep.out_row_dev) ep.out = static_cast<char*>(ep.out) + (long long)*ep.out_row_dev * ep.out_row_bytes;
    if (LN) {
        for (int m = wib; m < MM; m += GV_WARPS) ln_row<T>(ln.x + (long long)m * K, ln.w, ln.b, K, xs + m * K, lane);
        __syncthreads();
    }
    bool first = true;
    for (int g = g0; g < groups; g += warps) {
        const int n0 = g * RG;
        if (!first) {
#pragma unroll
            for (int r = 0; r < RG; ++r) wr[r] = reinterpret_cast<const uint4*>(W + (long long)min(n0 + r, N - 1) * K);
        }
        float acc[RG][MM];
#pragma unroll
        for (int r = 0; r < RG; ++r)
#pragma unroll
            for (int m = 0; m < MM; ++m) acc[r][m] = 0.f;
        for (int j0 = lane; j0 < K16; j0 += 32 * U) {
            if (!first) load_w<T, RG, U>(wr, j0, K16, wq);
            first = false;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int j = j0 + 32 * u;
                if (j < K16) {
#pragma unroll
                    for (int m = 0; m < MM; ++m) {
                        float a[VE];
                        if (LN)
                            GvVec<T>::unpack(*reinterpret_cast<const uint4*>(xs + (long long)m * K + j * VE), a);
                        else
                            GvVec<T>::unpack(__ldg(reinterpret_cast<const uint4*>(x + (long long)m * K) + j), a);
#pragma unroll
                        for (int r = 0; r < RG; ++r) {
                            float w[VE];
                            GvVec<T>::unpack(wq[r][u], w);
#pragma unroll
                            for (int e = 0; e < VE; ++e) acc[r][m] = fmaf(a[e], w[e], acc[r][m]);
                        }
                    }
                }
            }
        }
        first = false;
#pragma unroll
        for (int r = 0; r < RG; ++r)
#pragma unroll
            for (int m = 0; m < MM; ++m) acc[r][m] = warp_sum(acc[r][m]);
        // lane r*MM + m applies the epilogue to output (m, n0 + r)
#pragma unroll
        for (int r = 0; r < RG; ++r)
#pragma unroll
            for (int m = 0; m < MM; ++m)
                if (lane == r * MM + m && n0 + r < N) epilogue_scalar<T>(ep, m, n0 + r, 1, &acc[r][m]);
    }
}

template <typename T, int MM, int RG, int U>
void launch_rg(const Ctx& ctx, const T* x, const T* W, int N, int K, const Epilogue& ep, const LnIn& ln) {
    const int groups = ceil_div(N, RG);
    const int sms = ctx.num_sms > 0 ? ctx.num_sms : 148;
    const int blocks = std::min(ceil_div(groups, GV_WARPS), 8 * sms);
    if (ln.x) {
        const size_t smem = (size_t)MM * K * sizeof(T);
        launch_pdl(ctx, gemv_kernel<T, MM, RG, U, true>, dim3(blocks), dim3(GV_THREADS), smem, x, W, N, K, ep, ln);
    } else {
        launch_pdl(ctx, gemv_kernel<T, MM, RG, U, false>, dim3(blocks), dim3(GV_THREADS), 0, x, W, N, K, ep, ln);
    }
}

// Rows per group RG and steps per lane U (RG * U <= 16 loads of 16 bytes in
// flight per lane): short rows (at most 4 steps a lane) take 4 rows a group
// while that leaves four groups per SM, else 2, else 1; longer rows take U = 8
// (at most 8 steps) or 16 with 1 or 2 rows.
template <typename T, int MM>
void launch_mm(const Ctx& ctx, const T* x, const T* W, int N, int K, const Epilogue& ep, const LnIn& ln) {
    const int sms = ctx.num_sms > 0 ? ctx.num_sms : 148;
    const int per_lane = ceil_div(K / GvVec<T>::N, 32);
    if (per_lane <= 4) {
        if (N >= 4 * 4 * sms) launch_rg<T, MM, 4, 4>(ctx, x, W, N, K, ep, ln);
        else if (N >= 2 * 4 * sms) launch_rg<T, MM, 2, 4>(ctx, x, W, N, K, ep, ln);
        else launch_rg<T, MM, 1, 4>(ctx, x, W, N, K, ep, ln);
    } else if (per_lane <= 8) {
        if (N >= 2 * 4 * sms) launch_rg<T, MM, 2, 8>(ctx, x, W, N, K, ep, ln);
        else launch_rg<T, MM, 1, 8>(ctx, x, W, N, K, ep, ln);
    } else {
        launch_rg<T, MM, 1, 16>(ctx, x, W, N, K, ep, ln);
    }
}

}  // namespace

bool gemv_supported(size_t elem_size, int M, int K) {
    return M >= 1 && M <= GEMV_MAX_M && K >= 1 && (K * elem_size) % 16 == 0;
}

template <typename T>
void launch_gemv(const Ctx& ctx, const T* x, const T* W, int M, int N, int K, const Epilogue& ep, const LnIn& ln) {
    switch (M) {
    case 1: launch_mm<T, 1>(ctx, x, W, N, K, ep, ln); break;
    case 2: launch_mm<T, 2>(ctx, x, W, N, K, ep, ln); break;
    case 3: launch_mm<T, 3>(ctx, x, W, N, K, ep, ln); break;
    default: launch_mm<T, 4>(ctx, x, W, N, K, ep, ln); break;
    }
    ++*ctx.launches;
}

template void launch_gemv<float>(const Ctx&, const float*, const float*, int, int, int, const Epilogue&,
                                 const LnIn&);
template void launch_gemv<bf16>(const Ctx&, const bf16*, const bf16*, int, int, int, const Epilogue&, const LnIn&);

}  // namespace gpt2
