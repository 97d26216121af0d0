// Memory-bound row-wise kernels: embedding (+ first LayerNorm), LayerNorm
// forward/backward fused with the residual-gradient add and bias-gradient
// column sums, the cross-entropy classifier, column sums and the embedding
// backward scatter-add.
//
// Source definitions ("GPT-2 from Scratch"): "Embeddings: tokens and
// positions" (x = wte[idx] + wpe[t], positions from 0); "The Block: pre-LN and
// residuals" (nn.LayerNorm, eps 1e-5, biased variance); "Forward: logits, and
// loss when targets are given" (F.cross_entropy with ignore_index=-1);
// "Weight tying" (the embedding gradient lands in the same wte gradient as the
// lm_head weight gradient).
#include <algorithm>

#include "kernels.cuh"

namespace gpt2 {

namespace {

constexpr float LN_EPS = 1e-5f;


// A row of C floats spread over one warp: lane l holds float4 chunks
// l, l + 32, ..., i.e. columns 4*(l + 32 i) .. +3, for i < NV.
template <int NV>
struct RowFrag {
    float v[NV][4];
};

template <typename T, int NV, bool EMBED>
__global__ void __launch_bounds__(256) ln_fwd_kernel(const int* __restrict__ idx, const float* __restrict__ wte,
                                                      const float* __restrict__ wpe, int Tn, int V,
                                                      const float* __restrict__ x_in, const float* __restrict__ w,
                                                      const float* __restrict__ b, float* __restrict__ x_out,
                                                      T* __restrict__ y, float* __restrict__ mean,
                                                      float* __restrict__ rstd, int rows, int C, unsigned* status,
                                                      const int* __restrict__ pos_dev) {
    const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    griddep_launch();
    griddep_wait();
    if (row >= rows) return;
    float v[NV][4];
    const float* src;
    const float* src2 = nullptr;
    if (EMBED) {
        int tok = idx[row];
        if (tok < 0 || tok >= V) {
            if (lane == 0) atomicOr(status, STATUS_BAD_TOKEN);
            tok = tok < 0 ? 0 : V - 1;
        }
        src = wte + (long long)tok * C;
        src2 = wpe + (long long)((pos_dev ? *pos_dev : 0) + row % Tn) * C;
    } else {
        src = x_in + (long long)row * C;
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int c = (lane + 32 * i) * 4;
        if (c < C) {
            load4(src + c, v[i]);
            if (EMBED) {
                float p[4];
                load4(src2 + c, p);
#pragma unroll
                for (int j = 0; j < 4; ++j) v[i][j] += p[j];
                store4(x_out + (long long)row * C + c, v[i]);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) s += v[i][j];
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) v[i][j] = 0.f;
        }
    }
    const float mu = warp_sum(s) / C;
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int c = (lane + 32 * i) * 4;
        if (c < C) {
#pragma unroll
            for (int j = 0; j < 4; ++j) { float d = v[i][j] - mu; ss += d * d; }
        }
    }
    const float rs = rsqrtf(warp_sum(ss) / C + LN_EPS);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int c = (lane + 32 * i) * 4;
        if (c < C) {
            float ww[4], bb[4], o[4];
            load4(w + c, ww);
            load4(b + c, bb);
#pragma unroll
            for (int j = 0; j < 4; ++j) o[j] = (v[i][j] - mu) * rs * ww[j] + bb[j];
            store4(y + (long long)row * C + c, o);
        }
    }
    if (lane == 0) { mean[row] = mu; rstd[row] = rs; }
}

// LayerNorm backward, one pass over the rows. A warp per row computes
// dx = rstd (dxhat - mean(dxhat) - xhat mean(dxhat xhat)) + dres_in, dxhat = dy * w,
// and writes it as fp32 (residual gradient) and in the GEMM operand type. The
// same pass adds, per column, dy * xhat (weight gradient), dy (bias gradient)
// and dx (bias gradient of the GEMM that produced this LayerNorm's input) into
// the warp's own shared-memory row of partial sums (lane-owned columns, no
// atomics). At the end the block adds its 8 warp rows in a fixed order and
// writes one partial row per block; colred_finalize_kernel adds those
// (deterministic). Block b owns rows [b rows_per_block, (b + 1) rows_per_block).
constexpr int LNB_WARPS = 8;
template <typename T, int NV>
__global__ void __launch_bounds__(32 * LNB_WARPS, NV <= 8 ? 2 : 1)
    ln_bwd_kernel(const T* __restrict__ dy, const float* __restrict__ x, const float* __restrict__ mean,
                  const float* __restrict__ rstd, const float* __restrict__ w, const float* dres_in, float* dres_out,
                  T* __restrict__ dres_act, int rows, int C, int rows_per_block, int want_dx_sum,
                  float* __restrict__ partial) {
    extern __shared__ float4 acc4[];   // [LNB_WARPS][3][C / 4]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C4 = C >> 2;
    float4* mine = acc4 + warp * 3 * C4;
    for (int i = lane; i < 3 * C4; i += 32) mine[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    const int r0 = blockIdx.x * rows_per_block;
    const int r1 = min(rows, r0 + rows_per_block);
    for (int row = r0 + warp; row < r1; row += LNB_WARPS) {
        const float mu = mean[row], rs = rstd[row];
        float dxh[NV][4], xh[NV][4], res[NV][4];
        float s1 = 0.f, s2 = 0.f;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int c4 = lane + 32 * i;
            if (c4 < C4) {
                const int c = 4 * c4;
                float g[4], xx[4], ww[4];
                load4(dy + (long long)row * C + c, g);
                load4(x + (long long)row * C + c, xx);
                load4(w + c, ww);
                if (dres_in) load4(dres_in + (long long)row * C + c, res[i]);   // with the row's other loads
                else res[i][0] = res[i][1] = res[i][2] = res[i][3] = 0.f;
                float4 aw = mine[c4], ab = mine[C4 + c4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    xh[i][j] = (xx[j] - mu) * rs;
                    dxh[i][j] = g[j] * ww[j];
                    s1 += dxh[i][j];
                    s2 += dxh[i][j] * xh[i][j];
                }
                aw.x += g[0] * xh[i][0]; aw.y += g[1] * xh[i][1]; aw.z += g[2] * xh[i][2]; aw.w += g[3] * xh[i][3];
                ab.x += g[0]; ab.y += g[1]; ab.z += g[2]; ab.w += g[3];
                mine[c4] = aw;
                mine[C4 + c4] = ab;
            }
        }
        s1 = warp_sum(s1) / C;
        s2 = warp_sum(s2) / C;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int c4 = lane + 32 * i;
            if (c4 < C4) {
                const int c = 4 * c4;
                float o[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) o[j] = rs * (dxh[i][j] - s1 - xh[i][j] * s2) + res[i][j];
                store4(dres_out + (long long)row * C + c, o);
                if (dres_act) store4(dres_act + (long long)row * C + c, o);
                if (want_dx_sum) {
                    float4 an = mine[2 * C4 + c4];
                    an.x += o[0]; an.y += o[1]; an.z += o[2]; an.w += o[3];
                    mine[2 * C4 + c4] = an;
                }
            }
        }
    }
    __syncthreads();
    float4* part = reinterpret_cast<float4*>(partial + (long long)blockIdx.x * 3 * C);
    for (int i = threadIdx.x; i < 3 * C4; i += blockDim.x) {
        float4 t = acc4[i];
#pragma unroll
        for (int k = 1; k < LNB_WARPS; ++k) {
            const float4 u = acc4[k * 3 * C4 + i];
            t.x += u.x; t.y += u.y; t.z += u.z; t.w += u.w;
        }
        part[i] = t;
    }
}

// The same LayerNorm backward with each warp's next row (dy, x, dres_in) copied
// into a two-slot shared-memory ring by cp.async while the current row is
// processed, so every warp keeps a row of loads in flight. Shared memory:
// 8 warps x (3 partial rows + 2 ring rows) = 256 C bytes for bf16 dy, so
// C <= 880; one block per SM. Lane-owned columns: each lane reads back exactly
// the chunks it copied, so the ring needs no synchronisation across lanes.
__device__ __forceinline__ void cp_async_16(void* smem_dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_8(void* smem_dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit_group() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

constexpr int LNB_RING_BLOCKS = 148;   // one block per SM of a B200; a fixed count keeps the sum order fixed
// RING slots per warp (RING - 1 rows in flight ahead of the one processed). The
// column partial sums stay in registers (each lane owns its columns) and meet in
// shared memory, reusing the ring, once the block's rows are done.
template <typename T, int NV, int RING>
__global__ void __launch_bounds__(32 * LNB_WARPS, 1)
    ln_bwd_ring_kernel(const T* __restrict__ dy, const float* __restrict__ x, const float* __restrict__ mean,
                       const float* __restrict__ rstd, const float* __restrict__ w, const float* dres_in,
                       float* dres_out, T* __restrict__ dres_act, int rows, int C, int rows_per_block,
                       int want_dx_sum, float* __restrict__ partial) {
    extern __shared__ float4 smem4[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C4 = C >> 2;
    const size_t row_bytes = (size_t)C * (sizeof(T) + 8);   // dy | x | dres_in
    uint8_t* ring = reinterpret_cast<uint8_t*>(smem4) + (size_t)warp * RING * row_bytes;
    float ww[NV][4], aw[NV][4], ab[NV][4], an[NV][4];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int c4 = lane + 32 * i;
        if (c4 < C4) load4(w + 4 * c4, ww[i]);
#pragma unroll
        for (int j = 0; j < 4; ++j) aw[i][j] = ab[i][j] = an[i][j] = 0.f;
    }
    auto issue = [&](int row, int slot) {
        uint8_t* b = ring + slot * row_bytes;
        T* sdy = reinterpret_cast<T*>(b);
        float* sx = reinterpret_cast<float*>(b + (size_t)C * sizeof(T));
        float* sres = sx + C;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int c4 = lane + 32 * i;
            if (c4 < C4) {
                const long long g = (long long)row * C + 4 * c4;
                if (sizeof(T) == 2) cp_async_8(sdy + 4 * c4, dy + g);
                else cp_async_16(sdy + 4 * c4, dy + g);
                cp_async_16(sx + 4 * c4, x + g);
                if (dres_in) cp_async_16(sres + 4 * c4, dres_in + g);
            }
        }
        cp_async_commit_group();
    };
    const int r0 = blockIdx.x * rows_per_block;
    const int r1 = min(rows, r0 + rows_per_block);
#pragma unroll
    for (int k = 0; k < RING - 1; ++k)
        if (r0 + warp + k * LNB_WARPS < r1) issue(r0 + warp + k * LNB_WARPS, k);
    int slot = 0;
    for (int row = r0 + warp; row < r1; row += LNB_WARPS, slot = (slot + 1 == RING) ? 0 : slot + 1) {
        const float mu = mean[row], rs = rstd[row];
        // the row RING - 1 ahead into the slot processed last; then wait for this row's copies
        const int ahead = row + (RING - 1) * LNB_WARPS;
        if (ahead < r1) {
            issue(ahead, slot == 0 ? RING - 1 : slot - 1);
            cp_async_wait_group<RING - 1>();
        } else if (RING == 3 && row + LNB_WARPS < r1) {
            cp_async_wait_group<1>();
        } else {
            cp_async_wait_group<0>();
        }
        const uint8_t* b = ring + slot * row_bytes;
        const T* sdy = reinterpret_cast<const T*>(b);
        const float* sx = reinterpret_cast<const float*>(b + (size_t)C * sizeof(T));
        const float* sres = sx + C;
        float dxh[NV][4], xh[NV][4];
        float s1 = 0.f, s2 = 0.f;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int c4 = lane + 32 * i;
            if (c4 < C4) {
                float g[4], xx[4];
                load4(sdy + 4 * c4, g);
                load4(sx + 4 * c4, xx);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    xh[i][j] = (xx[j] - mu) * rs;
                    dxh[i][j] = g[j] * ww[i][j];
                    s1 += dxh[i][j];
                    s2 += dxh[i][j] * xh[i][j];
                    aw[i][j] += g[j] * xh[i][j];
                    ab[i][j] += g[j];
                }
            }
        }
        s1 = warp_sum(s1) / C;
        s2 = warp_sum(s2) / C;
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int c4 = lane + 32 * i;
            if (c4 < C4) {
                const int c = 4 * c4;
                float o[4], res[4] = {0.f, 0.f, 0.f, 0.f};
                if (dres_in) load4(sres + c, res);
#pragma unroll
                for (int j = 0; j < 4; ++j) o[j] = rs * (dxh[i][j] - s1 - xh[i][j] * s2) + res[j];
                store4(dres_out + (long long)row * C + c, o);
                if (dres_act) store4(dres_act + (long long)row * C + c, o);
                if (want_dx_sum) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) an[i][j] += o[j];
                }
            }
        }
    }
    __syncthreads();   // every warp is past its ring: the shared memory now holds the partial rows
    float4* acc4 = smem4;   // [LNB_WARPS][3][C / 4]
    float4* mine = acc4 + warp * 3 * C4;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int c4 = lane + 32 * i;
        if (c4 < C4) {
            mine[c4] = make_float4(aw[i][0], aw[i][1], aw[i][2], aw[i][3]);
            mine[C4 + c4] = make_float4(ab[i][0], ab[i][1], ab[i][2], ab[i][3]);
            mine[2 * C4 + c4] = make_float4(an[i][0], an[i][1], an[i][2], an[i][3]);
        }
    }
    __syncthreads();
    float4* part = reinterpret_cast<float4*>(partial + (long long)blockIdx.x * 3 * C);
    for (int i = threadIdx.x; i < 3 * C4; i += blockDim.x) {
        float4 t = acc4[i];
#pragma unroll
        for (int k = 1; k < LNB_WARPS; ++k) {
            const float4 u = acc4[k * 3 * C4 + i];
            t.x += u.x; t.y += u.y; t.z += u.z; t.w += u.w;
        }
        part[i] = t;
    }
}

// out_k[j] += sum over nblk partial rows of partial[b][k * n + j], k < n_out;
// a null out_k is skipped. Block = 32 columns x 32 row groups: each thread sums
// every 32nd partial row of its column (coalesced across the warp), then the
// 32 group sums are added in a fixed order (deterministic).
__global__ void __launch_bounds__(1024) colred_finalize_kernel(const float* __restrict__ partial, int nblk, int n,
                                                               int n_out, float* out0, float* out1, float* out2) {
    __shared__ float part[32][33];
    const int i = blockIdx.x * 32 + threadIdx.x;
    const int stride = n * n_out;
    float s = 0.f;
    if (i < stride) {
        // eight loads in flight per step; the additions keep their order
        int b = threadIdx.y;
        for (; b + 7 * 32 < nblk; b += 8 * 32) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = partial[(long long)(b + 32 * u) * stride + i];
#pragma unroll
            for (int u = 0; u < 8; ++u) s += v[u];
        }
        for (; b < nblk; b += 32) s += partial[(long long)b * stride + i];
    }
    part[threadIdx.y][threadIdx.x] = s;
    __syncthreads();
    if (threadIdx.y == 0 && i < stride) {
        float t = 0.f;
#pragma unroll
        for (int g = 0; g < 32; ++g) t += part[g][threadIdx.x];
        const int k = i / n, j = i % n;
        float* out = k == 0 ? out0 : (k == 1 ? out1 : out2);
        if (out) out[j] += t;
    }
}

__global__ void count_targets_kernel(const int* __restrict__ t, int n, int V, int* n_valid, unsigned* status) {
    __shared__ int cnt[32];
    int c = 0;
    bool bad = false;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int v = t[i];
        c += (v != -1);
        bad |= (v < -1 || v >= V);
    }
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(status, STATUS_BAD_TOKEN);
    if ((threadIdx.x & 31) == 0) cnt[threadIdx.x >> 5] = c;
    __syncthreads();
    if (threadIdx.x < 32) {
        int v = (threadIdx.x < (blockDim.x >> 5)) ? cnt[threadIdx.x] : 0;
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (threadIdx.x == 0) *n_valid = v;
    }
}

// Eight consecutive elements (16 bytes of bf16, 32 of fp32).
__device__ __forceinline__ void load8v(const float* p, float* v) { load4(p, v); load4(p + 4, v + 4); }
__device__ __forceinline__ void load8v(const bf16* p, float* v) {
    const uint4 q = *reinterpret_cast<const uint4*>(p);
    const unsigned u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[j]));
        v[2 * j] = f.x;
        v[2 * j + 1] = f.y;
    }
}
__device__ __forceinline__ void store8v(float* p, const float* v) { store4(p, v); store4(p + 4, v + 4); }
__device__ __forceinline__ void store8v(bf16* p, const float* v) {
    uint4 q;
    __nv_bfloat162 t[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) t[j] = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
    q.x = *reinterpret_cast<unsigned*>(&t[0]);
    q.y = *reinterpret_cast<unsigned*>(&t[1]);
    q.z = *reinterpret_cast<unsigned*>(&t[2]);
    q.w = *reinterpret_cast<unsigned*>(&t[3]);
    *reinterpret_cast<uint4*>(p) = q;
}
// exp for the softmax: CUDA's expf for fp32 logits, its fast __expf for bf16 logits.
template <typename T> __device__ __forceinline__ float sm_exp(float x);
template <> __device__ __forceinline__ float sm_exp<float>(float x) { return expf(x); }
template <> __device__ __forceinline__ float sm_exp<bf16>(float x) { return __expf(x); }

// One block per row. Pass 1: running max and sum of exp (online softmax) over
// all V columns; pass 2 (write_grad): dlogits = (softmax - onehot) * scale / n_valid,
// written in place; rows whose target is -1 get zeros. V is a multiple of 8.
template <typename T>
__global__ void __launch_bounds__(512) classifier_kernel(T* logits, const int* __restrict__ targets, int V,
                                                          const int* __restrict__ n_valid, float scale,
                                                          double* loss_accum, int write_grad) {
    const long long row = blockIdx.x;
    T* lr = logits + row * V;
    int tgt = targets[row];
    const bool valid = (tgt >= 0 && tgt < V);
    float lt = 0.f;
    if (threadIdx.x == 0 && valid) lt = to_f(lr[tgt]);
    float m = -INFINITY, s = 0.f;
    for (int c = threadIdx.x * 8; c < V; c += blockDim.x * 8) {
        float v[8];
        load8v(lr + c, v);
        float mx = v[0];
#pragma unroll
        for (int j = 1; j < 8; ++j) mx = fmaxf(mx, v[j]);
        if (mx > m) { s *= sm_exp<T>(m - mx); m = mx; }
#pragma unroll
        for (int j = 0; j < 8; ++j) s += sm_exp<T>(v[j] - m);
    }
    // block reduction of (m, s)
    __shared__ float sm[32], ssum[32];
    __shared__ float s_lse;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        float m2 = __shfl_xor_sync(0xffffffffu, m, o);
        float s2 = __shfl_xor_sync(0xffffffffu, s, o);
        float mm = fmaxf(m, m2);
        s = (m == -INFINITY ? 0.f : s * expf(m - mm)) + (m2 == -INFINITY ? 0.f : s2 * expf(m2 - mm));
        m = mm;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    if (lane == 0) { sm[warp] = m; ssum[warp] = s; }
    __syncthreads();
    if (warp == 0) {
        m = lane < nw ? sm[lane] : -INFINITY;
        s = lane < nw ? ssum[lane] : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            float m2 = __shfl_xor_sync(0xffffffffu, m, o);
            float s2 = __shfl_xor_sync(0xffffffffu, s, o);
            float mm = fmaxf(m, m2);
            s = (m == -INFINITY ? 0.f : s * expf(m - mm)) + (m2 == -INFINITY ? 0.f : s2 * expf(m2 - mm));
            m = mm;
        }
        if (lane == 0) s_lse = m + logf(s);
    }
    __syncthreads();
    const float lse = s_lse;
    const int nv = *n_valid;
    if (threadIdx.x == 0 && valid && nv > 0)
        atomicAdd(loss_accum, (double)scale * (double)(lse - lt) / (double)nv);
    if (!write_grad) return;
    const float gs = (valid && nv > 0) ? scale / (float)nv : 0.f;
    for (int c = threadIdx.x * 8; c < V; c += blockDim.x * 8) {
        float v[8];
        load8v(lr + c, v);
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = (sm_exp<T>(v[j] - lse) - (c + j == tgt ? 1.f : 0.f)) * gs;
        store8v(lr + c, v);
    }
}

// The classifier for bf16 logits: the same two passes with fewer instructions
// per element, since the fp32 version is issue-bound. The maximum of each
// 8-element chunk comes from packed bf16x2 max; exponentials are taken in
// log2 units, 2^(v log2(e) - m log2(e)), with one packed fma.f32x2 per pair
// and ex2.approx per element; sums and the gradient scale use packed pairs; the
// one target column of the row is patched after the chunk that holds it.
__device__ __forceinline__ void bf16x8_unpack(const uint4& q, f32x2 (&v)[4]) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[k]));
        v[k] = pk2(f.x, f.y);
    }
}
__global__ void __launch_bounds__(512) classifier_bf16_kernel(bf16* logits, const int* __restrict__ targets, int V,
                                                               const int* __restrict__ n_valid, float scale,
                                                               double* loss_accum, int write_grad) {
    constexpr float LOG2E = 1.4426950408889634f;
    const long long row = blockIdx.x;
    bf16* lr = logits + row * V;
    const int tgt = targets[row];
    const bool valid = (tgt >= 0 && tgt < V);
    float lt = 0.f;
    if (threadIdx.x == 0 && valid) lt = __bfloat162float(lr[tgt]);
    const f32x2 L2E = pk2(LOG2E, LOG2E);
    float m = -INFINITY;
    f32x2 S = pk2(0.f, 0.f);
    for (int c = threadIdx.x * 8; c < V; c += blockDim.x * 8) {
        const uint4 q = *reinterpret_cast<const uint4*>(lr + c);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
        const __nv_bfloat162 hm = __hmax2(__hmax2(h[0], h[1]), __hmax2(h[2], h[3]));
        const float mx = fmaxf(__low2float(hm), __high2float(hm));
        if (mx > m) {
            const float cr = ex2_approx((m - mx) * LOG2E);   // m = -inf at the start: 0
            S = mul2(S, pk2(cr, cr));
            m = mx;
        }
        const float nm = -m * LOG2E;
        const f32x2 NM = pk2(nm, nm);
        f32x2 v[4];
        bf16x8_unpack(q, v);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float t0, t1;
            upk2(fma2(v[k], L2E, NM), t0, t1);
            S = add2(S, pk2(ex2_approx(t0), ex2_approx(t1)));
        }
    }
    float s0, s1;
    upk2(S, s0, s1);
    float s = s0 + s1;
    // block reduction of (m, s)
    __shared__ float sm[32], ssum[32];
    __shared__ float s_lse;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        float m2 = __shfl_xor_sync(0xffffffffu, m, o);
        float s2 = __shfl_xor_sync(0xffffffffu, s, o);
        float mm = fmaxf(m, m2);
        s = (m == -INFINITY ? 0.f : s * expf(m - mm)) + (m2 == -INFINITY ? 0.f : s2 * expf(m2 - mm));
        m = mm;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    if (lane == 0) { sm[warp] = m; ssum[warp] = s; }
    __syncthreads();
    if (warp == 0) {
        m = lane < nw ? sm[lane] : -INFINITY;
        s = lane < nw ? ssum[lane] : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            float m2 = __shfl_xor_sync(0xffffffffu, m, o);
            float s2 = __shfl_xor_sync(0xffffffffu, s, o);
            float mm = fmaxf(m, m2);
            s = (m == -INFINITY ? 0.f : s * expf(m - mm)) + (m2 == -INFINITY ? 0.f : s2 * expf(m2 - mm));
            m = mm;
        }
        if (lane == 0) s_lse = m + logf(s);
    }
    __syncthreads();
    const float lse = s_lse;
    const int nv = *n_valid;
    if (threadIdx.x == 0 && valid && nv > 0)
        atomicAdd(loss_accum, (double)scale * (double)(lse - lt) / (double)nv);
    if (!write_grad) return;
    const float gs = (valid && nv > 0) ? scale / (float)nv : 0.f;
    const float nl = -lse * LOG2E;
    const f32x2 NL = pk2(nl, nl), GS = pk2(gs, gs);
    for (int c = threadIdx.x * 8; c < V; c += blockDim.x * 8) {
        const uint4 q = *reinterpret_cast<const uint4*>(lr + c);
        f32x2 v[4];
        bf16x8_unpack(q, v);
        float g[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float t0, t1;
            upk2(fma2(v[k], L2E, NL), t0, t1);
            upk2(mul2(pk2(ex2_approx(t0), ex2_approx(t1)), GS), g[2 * k], g[2 * k + 1]);
        }
        const int tj = tgt - c;
        if ((unsigned)tj < 8u) {   // the target column: softmax - 1
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (j == tj) g[j] -= gs;
        }
        store8v(lr + c, g);
    }
}

// Partial column sums of in[rows][cols] over blocks of rows: each thread owns 8
// consecutive columns and walks the block's rows with 16-byte loads.
template <typename T>
__global__ void colsum_partial_kernel(const T* __restrict__ in, int rows, int cols, int rows_per_block,
                                      float* __restrict__ partial) {
    const int col = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
    if (col >= cols) return;
    const int r0 = blockIdx.y * rows_per_block;
    const int r1 = min(rows, r0 + rows_per_block);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    int r = r0;
    for (; r + 8 <= r1; r += 8) {   // eight rows of loads in flight
        float v[8][8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            load4(in + (long long)(r + k) * cols + col, v[k]);
            load4(in + (long long)(r + k) * cols + col + 4, v[k] + 4);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] += v[k][j];
    }
    for (; r < r1; ++r) {
        float v[8];
        load4(in + (long long)r * cols + col, v);
        load4(in + (long long)r * cols + col + 4, v + 4);
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] += v[j];
    }
    float* p = partial + (long long)blockIdx.y * cols + col;
    store4(p, acc);
    store4(p + 4, acc + 4);
}

__global__ void embed_bwd_wte_kernel(const int* __restrict__ idx, const float* __restrict__ dx, int rows, int C,
                                     int V, float* dwte) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;   // float4 index
    const long long per_row = C / 4;
    if (i >= (long long)rows * per_row) return;
    const long long row = i / per_row;
    const int c = (int)(i % per_row) * 4;
    int tok = idx[row];
    tok = tok < 0 ? 0 : (tok >= V ? V - 1 : tok);
    float v[4];
    load4(dx + row * C + c, v);
    float* d = dwte + (long long)tok * C + c;
#pragma unroll
    for (int j = 0; j < 4; ++j) atomicAdd(d + j, v[j]);
}

// Deterministic embedding backward, per tile of at most EMB_TILE rows (tiles in
// row order). (1) Each block sorts one chunk of EMB_CHUNK packed keys
// (token << 16 | row in the tile) in shared memory (bitonic; the row breaks ties,
// so within a token the rows keep their order). (2) A warp per window of EMB_WIN
// sorted entries sums its rows, one piece per run of one token, in row order,
// into part[first position of the piece]; chunk ends are window ends. (3) A warp
// per run (a token's entries in one chunk) adds the run's pieces in position
// order into the run's first slot; then a warp per token adds its runs' sums in
// chunk order into dwte[token]. Chunks hold ascending rows, so each token's rows
// are added in row order, grouped; no atomics, every sum has a fixed order.
constexpr int EMB_TILE = 16384;
constexpr int EMB_CHUNK = 2048;
constexpr int EMB_WIN = 16;
static_assert(EMB_TILE <= 65536 && EMB_CHUNK % EMB_WIN == 0 && EMB_TILE / EMB_CHUNK <= 32, "emb tiling");

__global__ void __launch_bounds__(EMB_CHUNK / 2) emb_sort_kernel(const int* __restrict__ idx, int rows, int V,
                                                                 unsigned* __restrict__ sorted) {
    __shared__ unsigned ekey[EMB_CHUNK];
    const int base = blockIdx.x * EMB_CHUNK;
    for (int i = threadIdx.x; i < EMB_CHUNK; i += blockDim.x) {
        unsigned k = 0xFFFFFFFFu;   // padding sorts last
        if (base + i < rows) {
            int tok = idx[base + i];
            tok = tok < 0 ? 0 : (tok >= V ? V - 1 : tok);
            k = ((unsigned)tok << 16) | (unsigned)(base + i);
        }
        ekey[i] = k;
    }
    __syncthreads();
    const int t = threadIdx.x;   // one compare-exchange pair per thread and stage
    for (int k = 2; k <= EMB_CHUNK; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            const int i = 2 * t - (t & (j - 1));   // bit j of i is clear; the partner is i + j
            const unsigned a = ekey[i], b = ekey[i + j];
            if ((a > b) == ((i & k) == 0)) {
                ekey[i] = b;
                ekey[i + j] = a;
            }
            __syncthreads();
        }
    }
    for (int i = threadIdx.x; i < EMB_CHUNK && base + i < rows; i += blockDim.x) sorted[base + i] = ekey[i];
}

// Rows loaded together per batch (independent loads in flight), so that the
// buffer stays within the register file for the wider models.
template <int NV>
constexpr int emb_batch() { return NV <= 6 ? 4 : (NV <= 12 ? 2 : 1); }

template <int NV>
__global__ void __launch_bounds__(256) emb_piece_kernel(const unsigned* __restrict__ sorted, int n,
                                                        const float* __restrict__ dx, int C, float* __restrict__ part) {
    constexpr int U = emb_batch<NV>();
    const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    const int e0 = w * EMB_WIN;
    if (e0 >= n) return;
    const int cnt = min(EMB_WIN, n - e0);
    const unsigned mykey = lane < cnt ? sorted[e0 + lane] : 0xFFFFFFFFu;
    float acc[NV][4];
    auto clear = [&]() {
#pragma unroll
        for (int i = 0; i < NV; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    };
    auto store = [&](int pos) {
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int c = (lane + 32 * i) * 4;
            if (c < C) store4(part + (long long)pos * C + c, acc[i]);
        }
    };
    clear();
    int pstart = e0;
    unsigned tok_cur = __shfl_sync(0xffffffffu, mykey, 0) >> 16;
    for (int e = 0; e < cnt; e += U) {
        float v[U][NV][4];
        unsigned key[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            key[u] = __shfl_sync(0xffffffffu, mykey, e + u);
            if (e + u < cnt) {
                const float* src = dx + (long long)(key[u] & 0xFFFFu) * C;
#pragma unroll
                for (int i = 0; i < NV; ++i) {
                    const int c = (lane + 32 * i) * 4;
                    if (c < C) load4(src + c, v[u][i]);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (e + u < cnt) {
                if ((key[u] >> 16) != tok_cur) {   // a new run starts a new piece
                    store(pstart);
                    clear();
                    pstart = e0 + e + u;
                    tok_cur = key[u] >> 16;
                }
#pragma unroll
                for (int i = 0; i < NV; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] += v[u][i][j];
            }
        }
    }
    store(pstart);
}

// (3a) A warp per run (a token's entries inside one chunk) adds the run's pieces in
// position order and leaves the run's sum in the slot of its first piece.
template <int NV>
__global__ void __launch_bounds__(256) emb_run_kernel(const unsigned* __restrict__ sorted, int n,
                                                      float* __restrict__ part, int C) {
    constexpr int U = emb_batch<NV>();
    const int p = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (p >= n) return;
    const int chunk = p / EMB_CHUNK;
    const unsigned tok = sorted[p] >> 16;
    if (p > chunk * EMB_CHUNK && (sorted[p - 1] >> 16) == tok) return;   // not the start of a run
    const int cend = min(n, (chunk + 1) * EMB_CHUNK);
    const int b1 = (p / EMB_WIN + 1) * EMB_WIN;   // the run's later pieces start at window boundaries
    if (b1 >= cend || (sorted[b1] >> 16) != tok) return;   // one piece: already the run's sum
    float acc[NV][4];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int c = (lane + 32 * i) * 4;
        if (c < C) load4(part + (long long)p * C + c, acc[i]);
    }
    for (int q = b1; q < cend && (sorted[q] >> 16) == tok; q += U * EMB_WIN) {
        float v[U][NV][4];
        bool ok[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int qu = q + u * EMB_WIN;
            ok[u] = u == 0 || (ok[u - 1] && qu < cend && (sorted[qu] >> 16) == tok);
            if (ok[u]) {
#pragma unroll
                for (int i = 0; i < NV; ++i) {
                    const int c = (lane + 32 * i) * 4;
                    if (c < C) load4(part + (long long)qu * C + c, v[u][i]);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (ok[u]) {
#pragma unroll
                for (int i = 0; i < NV; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] += v[u][i][j];
            }
        }
        if (!ok[U - 1]) break;
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int c = (lane + 32 * i) * 4;
        if (c < C) store4(part + (long long)p * C + c, acc[i]);
    }
}

// (3b) A warp per run finds, by a binary search per chunk (one lane each), where
// its token's run starts in every chunk; the warp of the token's first chunk adds
// the runs' sums in chunk order into dwte[token].
template <int NV>
__global__ void __launch_bounds__(256) emb_token_kernel(const unsigned* __restrict__ sorted, int n,
                                                        const float* __restrict__ part, int C,
                                                        float* __restrict__ dwte) {
    const int p = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (p >= n) return;
    const int chunk = p / EMB_CHUNK;
    const unsigned tok = sorted[p] >> 16;
    if (p > chunk * EMB_CHUNK && (sorted[p - 1] >> 16) == tok) return;   // not the start of a run
    const int nch = (n + EMB_CHUNK - 1) / EMB_CHUNK;
    int start = -1;   // lane c: where the token's run starts in chunk c (lower bound of tok << 16)
    if (lane < nch && lane != chunk) {
        int lo = lane * EMB_CHUNK, hi = min(n, lo + EMB_CHUNK);
        const int end = hi;
        const unsigned key = tok << 16;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (sorted[mid] < key) lo = mid + 1;
            else hi = mid;
        }
        if (lo < end && (sorted[lo] >> 16) == tok) start = lo;
    }
    if (lane == chunk) start = p;
    const unsigned present = __ballot_sync(0xffffffffu, start >= 0);
    if ((int)(__ffs(present) - 1) != chunk) return;   // an earlier chunk's run owns the token
    float acc[NV][4];
#pragma unroll
    for (int i = 0; i < NV; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    float* d = dwte + (long long)tok * C;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int c = (lane + 32 * i) * 4;
        if (c < C) load4(d + c, acc[i]);
    }
    for (unsigned m = present; m; m &= m - 1) {
        const int q = __shfl_sync(0xffffffffu, start, __ffs(m) - 1);
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            const int c = (lane + 32 * i) * 4;
            if (c < C) {
                float v[4];
                load4(part + (long long)q * C + c, v);
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] += v[j];
            }
        }
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int c = (lane + 32 * i) * 4;
        if (c < C) store4(d + c, acc[i]);
    }
}

template <int NV>
void emb_tile(const Ctx& ctx, const int* idx, const float* dx, int rows, int C, int V, float* dwte, float* part,
              unsigned* sorted) {
    emb_sort_kernel<<<ceil_div(rows, EMB_CHUNK), EMB_CHUNK / 2, 0, ctx.stream>>>(idx, rows, V, sorted);
    const int windows = ceil_div(rows, EMB_WIN);
    emb_piece_kernel<NV><<<ceil_div(windows, 8), 256, 0, ctx.stream>>>(sorted, rows, dx, C, part);
    emb_run_kernel<NV><<<ceil_div(rows, 8), 256, 0, ctx.stream>>>(sorted, rows, part, C);
    emb_token_kernel<NV><<<ceil_div(rows, 8), 256, 0, ctx.stream>>>(sorted, rows, part, C, dwte);
    *ctx.launches += 4;
}

__global__ void embed_bwd_wpe_kernel(const float* __restrict__ dx, int B, int Tn, int C, float* dwpe) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)Tn * C) return;
    float s = 0.f;
    for (int b = 0; b < B; ++b) s += dx[(long long)b * Tn * C + i];
    dwpe[i] += s;
}

template <typename T, bool EMBED>
void ln_fwd_dispatch(const Ctx& ctx, const int* idx, const float* wte, const float* wpe, int Tn, int V,
                     const float* x_in, const float* w, const float* b, float* x_out, T* y, float* mean,
                     float* rstd, int rows, int C, const int* pos_dev) {
    const int threads = 256;
    const int blocks = ceil_div(rows, threads / 32);
    const int nv = ceil_div(C, 128);
#define LNF_CASE(N)                                                                                 \
    case N:                                                                                         \
        launch_pdl(ctx, ln_fwd_kernel<T, N, EMBED>, dim3(blocks), dim3(threads), 0, idx, wte, wpe, Tn, V, \
                   x_in, w, b, x_out, y, mean, rstd, rows, C, ctx.status, pos_dev);                     \
        break;
    switch (nv) {
        LNF_CASE(1) LNF_CASE(2) LNF_CASE(3) LNF_CASE(4) LNF_CASE(5) LNF_CASE(6) LNF_CASE(7)
        LNF_CASE(8) LNF_CASE(9) LNF_CASE(10) LNF_CASE(11) LNF_CASE(12) LNF_CASE(13) LNF_CASE(14)
        LNF_CASE(15) LNF_CASE(16)
        default: break;
    }
#undef LNF_CASE
    ++*ctx.launches;
}

}  // namespace

template <typename T>
void launch_embed_ln(const Ctx& ctx, const int* idx, const float* wte, const float* wpe, int rows, int Tn, int C,
                     int V, const float* w, const float* b, float* x, T* y, float* mean, float* rstd,
                     const int* pos_dev) {
    ln_fwd_dispatch<T, true>(ctx, idx, wte, wpe, Tn, V, nullptr, w, b, x, y, mean, rstd, rows, C, pos_dev);
}

template <typename T>
void launch_layernorm_fwd(const Ctx& ctx, const float* x, const float* w, const float* b, T* y, float* mean,
                          float* rstd, int rows, int C) {
    ln_fwd_dispatch<T, false>(ctx, nullptr, nullptr, nullptr, 1, 1, x, w, b, nullptr, y, mean, rstd, rows, C,
                              nullptr);
}

template <typename T>
void launch_layernorm_bwd(const Ctx& ctx, const T* dy, const float* x, const float* mean, const float* rstd,
                          const float* w, const float* dres_in, float* dres_out, T* dres_act, float* dw,
                          float* db, float* dbias_next, int rows, int C, float* scratch) {
    const int nv = ceil_div(C, 128);
    const int want = dbias_next != nullptr;
    // shared memory: the ring (RING rows per warp), reused for the partial rows at the end
    const size_t row_bytes = (size_t)C * (sizeof(T) + 8), parts = (size_t)LNB_WARPS * 3 * C * sizeof(float);
    const size_t ring3 = std::max((size_t)LNB_WARPS * 3 * row_bytes, parts);
    const size_t ring2 = std::max((size_t)LNB_WARPS * 2 * row_bytes, parts);
    const int ring = ring3 <= 220 * 1024 ? 3 : 2;
    const size_t ring_smem = ring == 3 ? ring3 : ring2;
    if (ring_smem <= 220 * 1024 && nv <= 8) {
        const int nblk = min(ceil_div(rows, LNB_WARPS), LNB_RING_BLOCKS);
        const int rpb = ceil_div(rows, nblk);
#define LNR_CASE(N)                                                                                         \
    case N: {                                                                                               \
        static bool configured = false;                                                                     \
        if (!configured) {                                                                                  \
            cudaFuncSetAttribute(ln_bwd_ring_kernel<T, N, 3>, cudaFuncAttributeMaxDynamicSharedMemorySize,  \
                                 220 * 1024);                                                               \
            cudaFuncSetAttribute(ln_bwd_ring_kernel<T, N, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,  \
                                 220 * 1024);                                                               \
            configured = true;                                                                              \
        }                                                                                                   \
        if (ring == 3)                                                                                      \
            ln_bwd_ring_kernel<T, N, 3><<<nblk, 32 * LNB_WARPS, ring_smem, ctx.stream>>>(                   \
                dy, x, mean, rstd, w, dres_in, dres_out, dres_act, rows, C, rpb, want, scratch);            \
        else                                                                                                \
            ln_bwd_ring_kernel<T, N, 2><<<nblk, 32 * LNB_WARPS, ring_smem, ctx.stream>>>(                   \
                dy, x, mean, rstd, w, dres_in, dres_out, dres_act, rows, C, rpb, want, scratch);            \
        break;                                                                                              \
    }
        switch (nv) {
            LNR_CASE(1) LNR_CASE(2) LNR_CASE(3) LNR_CASE(4) LNR_CASE(5) LNR_CASE(6) LNR_CASE(7) LNR_CASE(8)
            default: break;
        }
#undef LNR_CASE
        colred_finalize_kernel<<<ceil_div(3 * C, 32), dim3(32, 32), 0, ctx.stream>>>(scratch, nblk, C, 3, dw, db,
                                                                                      dbias_next);
        *ctx.launches += 2;
        return;
    }
    const int nblk = ln_bwd_col_blocks(rows);
    const int rpb = ceil_div(rows, nblk);
    const size_t smem = (size_t)LNB_WARPS * 3 * C * sizeof(float);
#define LNB_CASE(N)                                                                                         \
    case N: {                                                                                               \
        static bool configured = false;                                                                     \
        if (!configured) {                                                                                  \
            cudaFuncSetAttribute(ln_bwd_kernel<T, N>, cudaFuncAttributeMaxDynamicSharedMemorySize,          \
                                 (int)(LNB_WARPS * 3 * 128 * N * sizeof(float)));                           \
            cudaFuncSetAttribute(ln_bwd_kernel<T, N>, cudaFuncAttributePreferredSharedMemoryCarveout, 100); \
            configured = true;                                                                              \
        }                                                                                                   \
        ln_bwd_kernel<T, N><<<nblk, 32 * LNB_WARPS, smem, ctx.stream>>>(dy, x, mean, rstd, w, dres_in,      \
                                                                        dres_out, dres_act, rows, C, rpb,   \
                                                                        want, scratch);                     \
        break;                                                                                              \
    }
    switch (nv) {
        LNB_CASE(1) LNB_CASE(2) LNB_CASE(3) LNB_CASE(4) LNB_CASE(5) LNB_CASE(6) LNB_CASE(7)
        LNB_CASE(8) LNB_CASE(9) LNB_CASE(10) LNB_CASE(11) LNB_CASE(12) LNB_CASE(13) LNB_CASE(14)
        LNB_CASE(15) LNB_CASE(16)
        default: break;
    }
#undef LNB_CASE
    colred_finalize_kernel<<<ceil_div(3 * C, 32), dim3(32, 32), 0, ctx.stream>>>(scratch, nblk, C, 3, dw, db,
                                                                                  dbias_next);
    *ctx.launches += 2;
}

void launch_colred_finalize(const Ctx& ctx, const float* partial, int nblk, int n, float* out) {
    colred_finalize_kernel<<<ceil_div(n, 32), dim3(32, 32), 0, ctx.stream>>>(partial, nblk, n, 1, out, nullptr,
                                                                              nullptr);
    ++*ctx.launches;
}

template <typename T>
__global__ void gather_last_rows_kernel(const T* __restrict__ src, int Tn, int C, T* __restrict__ dst) {
    const int b = blockIdx.x;
    const uint4* s = reinterpret_cast<const uint4*>(src + ((long long)b * Tn + Tn - 1) * C);
    uint4* d = reinterpret_cast<uint4*>(dst + (long long)b * C);
    for (int i = threadIdx.x; i < C * (int)sizeof(T) / 16; i += blockDim.x) d[i] = s[i];
}

template <typename T>
void launch_gather_last_rows(const Ctx& ctx, const T* src, int B, int Tn, int C, T* dst) {
    gather_last_rows_kernel<T><<<B, 128, 0, ctx.stream>>>(src, Tn, C, dst);
    ++*ctx.launches;
}

void launch_count_targets(const Ctx& ctx, const int* targets, int n, int V, int* n_valid) {
    count_targets_kernel<<<1, 1024, 0, ctx.stream>>>(targets, n, V, n_valid, ctx.status);
    ++*ctx.launches;
}

template <typename T>
void launch_classifier(const Ctx& ctx, T* logits, const int* targets, int rows, int V, const int* n_valid,
                       float scale, double* loss_accum, int write_grad) {
    if (sizeof(T) == 2)
        classifier_bf16_kernel<<<rows, 512, 0, ctx.stream>>>(reinterpret_cast<bf16*>(logits), targets, V, n_valid,
                                                              scale, loss_accum, write_grad);
    else
        classifier_kernel<T><<<rows, 512, 0, ctx.stream>>>(logits, targets, V, n_valid, scale, loss_accum, write_grad);
    ++*ctx.launches;
}

template <typename T>
void launch_colsum(const Ctx& ctx, const T* in, int rows, int cols, float* out, float* scratch) {
    const int nblk = colsum_row_blocks(rows);
    const int rpb = ceil_div(rows, nblk);
    dim3 grid(ceil_div(cols, 8 * 64), nblk);   // many small blocks: enough loads in flight on every SM
    colsum_partial_kernel<T><<<grid, 64, 0, ctx.stream>>>(in, rows, cols, rpb, scratch);
    colred_finalize_kernel<<<ceil_div(cols, 32), dim3(32, 32), 0, ctx.stream>>>(scratch, nblk, cols, 1, out,
                                                                                nullptr, nullptr);
    *ctx.launches += 2;
}

void launch_embed_bwd(const Ctx& ctx, const int* idx, const float* dx, int B, int Tn, int C, int V, float* dwte,
                      float* dwpe, float* scratch) {
    const long long rows = (long long)B * Tn;
    const int nv = ceil_div(C, 128);
    if (scratch && V <= 65536 && nv <= 16 && C % 4 == 0) {
        float* part = scratch;
        unsigned* sorted = reinterpret_cast<unsigned*>(scratch + rows * C);
        for (long long r0 = 0; r0 < rows; r0 += EMB_TILE) {   // tiles in row order
            const int n = (int)std::min<long long>(EMB_TILE, rows - r0);
            const int* ti = idx + r0;
            const float* td = dx + r0 * C;
#define EMB_CASE(NV) \
    case NV: emb_tile<NV>(ctx, ti, td, n, C, V, dwte, part, sorted); break;
            switch (nv) {
                EMB_CASE(1) EMB_CASE(2) EMB_CASE(3) EMB_CASE(4) EMB_CASE(5) EMB_CASE(6) EMB_CASE(7) EMB_CASE(8)
                EMB_CASE(9) EMB_CASE(10) EMB_CASE(11) EMB_CASE(12) EMB_CASE(13) EMB_CASE(14) EMB_CASE(15)
                EMB_CASE(16)
                default: break;
            }
#undef EMB_CASE
        }
    } else {
        const long long n4 = rows * (C / 4);
        embed_bwd_wte_kernel<<<(unsigned)ceil_div_ll(n4, 256), 256, 0, ctx.stream>>>(idx, dx, (int)rows, C, V, dwte);
        ++*ctx.launches;
    }
    embed_bwd_wpe_kernel<<<(unsigned)ceil_div_ll((long long)Tn * C, 256), 256, 0, ctx.stream>>>(dx, B, Tn, C, dwpe);
    ++*ctx.launches;
}

#define INST(T)                                                                                                 \
    template void launch_embed_ln<T>(const Ctx&, const int*, const float*, const float*, int, int, int, int,   \
                                     const float*, const float*, float*, T*, float*, float*, const int*);      \
    template void launch_layernorm_fwd<T>(const Ctx&, const float*, const float*, const float*, T*, float*,    \
                                          float*, int, int);                                                   \
    template void launch_layernorm_bwd<T>(const Ctx&, const T*, const float*, const float*, const float*,      \
                                          const float*, const float*, float*, T*, float*, float*, float*, int, \
                                          int, float*);                                                        \
    template void launch_classifier<T>(const Ctx&, T*, const int*, int, int, const int*, float, double*, int); \
    template void launch_colsum<T>(const Ctx&, const T*, int, int, float*, float*);                          \
    template void launch_gather_last_rows<T>(const Ctx&, const T*, int, int, int, T*);
INST(float)
INST(bf16)
#undef INST

}  // namespace gpt2
