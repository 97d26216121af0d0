// Tensor-core causal flash attention (bf16 operands, fp32 accumulation and
// softmax), forward and backward, for head widths 32 and 64.
//
// Definitions ("GPT-2 from Scratch", "CausalSelfAttention"): q, k, v are the
// three C-wide column blocks of the fused qkv rows; head h owns columns
// [h*hd, (h+1)*hd) of each block; S = q k^T / sqrt(hd) with future keys masked
// to -inf; P = softmax(S); y = P v, heads concatenated in head order. The
// forward never stores S or P ("Let's reproduce GPT-2 (124M)", "FlashAttention
// and vocabulary padding": online softmax with a running max and sum); it keeps
// the row log-sum-exp for the backward, which recomputes P = exp(S - lse).
//
// Backward (D = rowsum(dO * O)):  dV = P^T dO,  dP = dO V^T,
//   dS = P * (dP - D),  dQ = dS K / sqrt(hd),  dK = dS^T Q / sqrt(hd).
// Two kernels: one per 64-key tile computes dK, dV from S^T = K Q^T (so every
// MMA operand is either already in registers or loaded by ldmatrix, with no
// shared-memory transposes and no atomics); one per 64-query tile computes dQ.
//
// Tiles: 64 rows per CTA, 16 rows per warp (4 warps), 64-column K/V or Q/dO
// tiles double-buffered with cp.async; MMA = mma.sync m16n8k16 (bf16 -> fp32).
#include "kernels.cuh"

namespace gpt2 {

namespace {

constexpr int TILE = 64;
constexpr int NTHR = 128;
constexpr float LOG2E = 1.4426950408889634f;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    const int sz = valid ? 16 : 0;   // 0: zero-fill, nothing read
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(sz) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t* r, uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t* r, uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Shared-memory tile of 64 rows x HD bf16 with a padded row stride (HD + 8
// elements) so that ldmatrix row addresses fall in distinct banks.
template <int HD>
struct Tile {
    static constexpr int STRIDE = HD + 8;
    static constexpr int BYTES = TILE * STRIDE * 2;
};

// Copy rows [row0, row0 + 64) x HD columns starting at `base + row * ld` into a
// tile; rows at or beyond Tn are zero-filled.
template <int HD>
__device__ __forceinline__ void load_tile(bf16* dst, const bf16* base, long long ld, int row0, int Tn) {
    constexpr int CPR = HD / 8;   // 16-byte chunks per row
#pragma unroll
    for (int i = threadIdx.x; i < TILE * CPR; i += NTHR) {
        const int r = i / CPR, c = i % CPR;
        const bool valid = row0 + r < Tn;
        const bf16* src = valid ? base + (long long)(row0 + r) * ld + c * 8 : base;
        cp_async16(smem_addr(dst + r * Tile<HD>::STRIDE + c * 8), src, valid);
    }
}

// A fragments (16 rows x HD) of rows [r0, r0+16) of a tile, kept in registers.
template <int HD>
__device__ __forceinline__ void load_a_frags(uint32_t (*frag)[4], const bf16* tile, int r0) {
    const int t = threadIdx.x & 31;
#pragma unroll
    for (int kc = 0; kc < HD / 16; ++kc) {
        const int row = r0 + (t & 7) + ((t >> 3) & 1) * 8;
        const int col = kc * 16 + (t >> 4) * 8;
        ldsm_x4(frag[kc], smem_addr(tile + row * Tile<HD>::STRIDE + col));
    }
}

// acc[nt] (16 x 64 over 8 n-tiles) += A(16 x HD, registers) * Rows^T where the
// tile holds 64 rows (the n index) x HD (the k index): B fragments by ldmatrix.
template <int HD>
__device__ __forceinline__ void mma_a_rowsT(float (*acc)[4], const uint32_t (*a)[4], const bf16* tile) {
    const int t = threadIdx.x & 31;
#pragma unroll
    for (int kc = 0; kc < HD / 16; ++kc) {
#pragma unroll
        for (int np = 0; np < 4; ++np) {
            uint32_t b[4];
            const int row = np * 16 + (t & 7) + (t >> 4) * 8;
            const int col = kc * 16 + ((t >> 3) & 1) * 8;
            ldsm_x4(b, smem_addr(tile + row * Tile<HD>::STRIDE + col));
            mma16816(acc[2 * np], a[kc], b[0], b[1]);
            mma16816(acc[2 * np + 1], a[kc], b[2], b[3]);
        }
    }
}

// acc[dt] (16 x HD) += P(16 x 64, as C fragments p[8][4] converted to A) * Rows
// where the tile holds 64 rows (the k index) x HD (the n index): ldmatrix.trans.
template <int HD>
__device__ __forceinline__ void mma_p_rows(float (*acc)[4], const float (*p)[4], const bf16* tile) {
    const int t = threadIdx.x & 31;
#pragma unroll
    for (int kc = 0; kc < 4; ++kc) {
        uint32_t a[4];
        a[0] = pack_bf16(p[2 * kc][0], p[2 * kc][1]);
        a[1] = pack_bf16(p[2 * kc][2], p[2 * kc][3]);
        a[2] = pack_bf16(p[2 * kc + 1][0], p[2 * kc + 1][1]);
        a[3] = pack_bf16(p[2 * kc + 1][2], p[2 * kc + 1][3]);
#pragma unroll
        for (int dp = 0; dp < HD / 16; ++dp) {
            uint32_t b[4];
            const int row = kc * 16 + (t & 7) + ((t >> 3) & 1) * 8;
            const int col = dp * 16 + (t >> 4) * 8;
            ldsm_x4_t(b, smem_addr(tile + row * Tile<HD>::STRIDE + col));
            mma16816(acc[2 * dp], a, b[0], b[1]);
            mma16816(acc[2 * dp + 1], a, b[2], b[3]);
        }
    }
}

template <int N>
__device__ __forceinline__ void zero(float (*acc)[4]) {
#pragma unroll
    for (int i = 0; i < N; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
}

// ============================================================== forward
template <int HD>
__global__ void __launch_bounds__(NTHR) flash_fwd_kernel(const bf16* __restrict__ qkv, bf16* __restrict__ out,
                                                        float* __restrict__ lse, int Tn, int H) {
    __shared__ __align__(16) bf16 Qs[TILE * Tile<HD>::STRIDE];
    __shared__ __align__(16) bf16 Ks[2][TILE * Tile<HD>::STRIDE];
    __shared__ __align__(16) bf16 Vs[2][TILE * Tile<HD>::STRIDE];
    const int qt = gridDim.x - 1 - blockIdx.x;   // longest rows first
    const int bh = blockIdx.y, b = bh / H, h = bh % H;
    const int C = H * HD;
    const long long ld = 3LL * C;
    const bf16* base = qkv + (long long)b * Tn * ld + h * HD;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q0 = qt * TILE;
    const float sl2 = LOG2E * rsqrtf((float)HD);

    load_tile<HD>(Qs, base, ld, q0, Tn);
    load_tile<HD>(Ks[0], base + C, ld, 0, Tn);
    load_tile<HD>(Vs[0], base + 2 * C, ld, 0, Tn);
    cp_async_commit();

    uint32_t qf[HD / 16][4];
    float o[HD / 8][4];
    zero<HD / 8>(o);
    float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
    const int row_g = q0 + warp * 16 + (lane >> 2);   // query of c0/c1; +8 for c2/c3

    const int n_kt = qt + 1;
    for (int kt = 0; kt < n_kt; ++kt) {
        const int buf = kt & 1;
        if (kt + 1 < n_kt) {
            load_tile<HD>(Ks[buf ^ 1], base + C, ld, (kt + 1) * TILE, Tn);
            load_tile<HD>(Vs[buf ^ 1], base + 2 * C, ld, (kt + 1) * TILE, Tn);
        }
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        if (kt == 0) load_a_frags<HD>(qf, Qs, warp * 16);

        float s[8][4];
        zero<8>(s);
        mma_a_rowsT<HD>(s, qf, Ks[buf]);
        const bool diag = (kt == qt);
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float v = s[nt][e] * sl2;
                if (diag) {
                    const int key = kt * TILE + nt * 8 + 2 * (lane & 3) + (e & 1);
                    const int q = row_g + (e >> 1) * 8;
                    if (key > q) v = -INFINITY;
                }
                s[nt][e] = v;
                mx[e >> 1] = fmaxf(mx[e >> 1], v);
            }
        }
        float corr[2];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
            mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
            const float mn = fmaxf(m_r[r], mx[r]);
            corr[r] = exp2f(m_r[r] - mn);   // m_r = -inf at the start: corr = 0
            m_r[r] = mn;
            l_r[r] *= corr[r];
        }
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float p = exp2f(s[nt][e] - m_r[e >> 1]);
                s[nt][e] = p;
                l_r[e >> 1] += p;
            }
        }
#pragma unroll
        for (int dt = 0; dt < HD / 8; ++dt) {
            o[dt][0] *= corr[0];
            o[dt][1] *= corr[0];
            o[dt][2] *= corr[1];
            o[dt][3] *= corr[1];
        }
        mma_p_rows<HD>(o, s, Vs[buf]);
        __syncthreads();
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 1);
        l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 2);
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int q = row_g + r * 8;
        if (q < Tn) {
            const float inv = 1.f / l_r[r];
            bf16* orow = out + ((long long)b * Tn + q) * C + h * HD;
#pragma unroll
            for (int dt = 0; dt < HD / 8; ++dt) {
                const int col = dt * 8 + 2 * (lane & 3);
                *reinterpret_cast<__nv_bfloat162*>(orow + col) =
                    __floats2bfloat162_rn(o[dt][2 * r] * inv, o[dt][2 * r + 1] * inv);
            }
            if ((lane & 3) == 0) lse[(long long)bh * Tn + q] = (m_r[r] + log2f(l_r[r])) / LOG2E;
        }
    }
}

// ================================================= backward: dK, dV per key tile
template <int HD>
__global__ void __launch_bounds__(NTHR) flash_bwd_dkv_kernel(const bf16* __restrict__ qkv,
                                                            const bf16* __restrict__ dout,
                                                            const float* __restrict__ lse,
                                                            const float* __restrict__ dpre,
                                                            bf16* __restrict__ dqkv, int Tn, int H) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    bf16* KVs = reinterpret_cast<bf16*>(smem_raw);                      // K tile then V tile
    bf16* Qs = KVs + 2 * TILE * Tile<HD>::STRIDE;                       // [2] Q tiles
    bf16* Ds = Qs + 2 * TILE * Tile<HD>::STRIDE;                        // [2] dO tiles
    float* Ls = reinterpret_cast<float*>(Ds + 2 * TILE * Tile<HD>::STRIDE);   // [2][64] lse (log2 units)
    float* Pd = Ls + 2 * TILE;                                          // [2][64] D
    const int kt = gridDim.x - 1 - blockIdx.x;
    const int bh = blockIdx.y, b = bh / H, h = bh % H;
    const int C = H * HD;
    const long long ld = 3LL * C;
    const bf16* base = qkv + (long long)b * Tn * ld + h * HD;
    const bf16* dobase = dout + (long long)b * Tn * C + h * HD;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int k0 = kt * TILE;
    const float sl2 = LOG2E * rsqrtf((float)HD);
    const int n_qt = (Tn + TILE - 1) / TILE;

    auto load_q = [&](int qt, int buf) {
        load_tile<HD>(Qs + buf * TILE * Tile<HD>::STRIDE, base, ld, qt * TILE, Tn);
        load_tile<HD>(Ds + buf * TILE * Tile<HD>::STRIDE, dobase, C, qt * TILE, Tn);
        if (threadIdx.x < TILE) {
            const int q = qt * TILE + threadIdx.x;
            Ls[buf * TILE + threadIdx.x] = q < Tn ? lse[(long long)bh * Tn + q] * LOG2E : INFINITY;
            Pd[buf * TILE + threadIdx.x] = q < Tn ? dpre[(long long)bh * Tn + q] : 0.f;
        }
    };
    load_tile<HD>(KVs, base + C, ld, k0, Tn);
    load_tile<HD>(KVs + TILE * Tile<HD>::STRIDE, base + 2 * C, ld, k0, Tn);
    load_q(kt, 0);
    cp_async_commit();

    uint32_t kf[HD / 16][4], vf[HD / 16][4];
    float dk[HD / 8][4], dv[HD / 8][4];
    zero<HD / 8>(dk);
    zero<HD / 8>(dv);
    const int key_g = k0 + warp * 16 + (lane >> 2);   // key of c0/c1 rows; +8 for c2/c3

    for (int qt = kt; qt < n_qt; ++qt) {
        const int buf = (qt - kt) & 1;
        if (qt + 1 < n_qt) load_q(qt + 1, buf ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        if (qt == kt) {
            load_a_frags<HD>(kf, KVs, warp * 16);
            load_a_frags<HD>(vf, KVs + TILE * Tile<HD>::STRIDE, warp * 16);
        }
        const bf16* Qt = Qs + buf * TILE * Tile<HD>::STRIDE;
        const bf16* Dt = Ds + buf * TILE * Tile<HD>::STRIDE;
        const float* Lt = Ls + buf * TILE;
        const float* Pt = Pd + buf * TILE;
        // S^T = K Q^T (16 keys x 64 queries per warp);  dP^T = V dO^T
        float st[8][4], dpt[8][4];
        zero<8>(st);
        zero<8>(dpt);
        mma_a_rowsT<HD>(st, kf, Qt);
        mma_a_rowsT<HD>(dpt, vf, Dt);
        const bool diag = (qt == kt);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int qi = nt * 8 + 2 * (lane & 3) + (e & 1);   // query within the tile
                float p = exp2f(st[nt][e] * sl2 - Lt[qi]);
                if (diag && (key_g + (e >> 1) * 8) > qt * TILE + qi) p = 0.f;
                st[nt][e] = p;                                           // P^T
                dpt[nt][e] = p * (dpt[nt][e] - Pt[qi]);                  // dS^T
            }
        }
        mma_p_rows<HD>(dv, st, Dt);    // dV += P^T dO
        mma_p_rows<HD>(dk, dpt, Qt);   // dK += dS^T Q
        __syncthreads();
    }
    const float scale = rsqrtf((float)HD);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int key = key_g + r * 8;
        if (key < Tn) {
            bf16* row = dqkv + ((long long)b * Tn + key) * ld + h * HD;
#pragma unroll
            for (int dt = 0; dt < HD / 8; ++dt) {
                const int col = dt * 8 + 2 * (lane & 3);
                *reinterpret_cast<__nv_bfloat162*>(row + C + col) =
                    __floats2bfloat162_rn(dk[dt][2 * r] * scale, dk[dt][2 * r + 1] * scale);
                *reinterpret_cast<__nv_bfloat162*>(row + 2 * C + col) =
                    __floats2bfloat162_rn(dv[dt][2 * r], dv[dt][2 * r + 1]);
            }
        }
    }
}

// ================================================ backward: dQ per query tile
template <int HD>
__global__ void __launch_bounds__(NTHR) flash_bwd_dq_kernel(const bf16* __restrict__ qkv,
                                                           const bf16* __restrict__ dout,
                                                           const float* __restrict__ lse,
                                                           const float* __restrict__ dpre,
                                                           bf16* __restrict__ dqkv, int Tn, int H) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    bf16* Qs = reinterpret_cast<bf16*>(smem_raw);
    bf16* Ds = Qs + TILE * Tile<HD>::STRIDE;
    bf16* Ks = Ds + TILE * Tile<HD>::STRIDE;   // [2]
    bf16* Vs = Ks + 2 * TILE * Tile<HD>::STRIDE;   // [2]
    const int qt = gridDim.x - 1 - blockIdx.x;
    const int bh = blockIdx.y, b = bh / H, h = bh % H;
    const int C = H * HD;
    const long long ld = 3LL * C;
    const bf16* base = qkv + (long long)b * Tn * ld + h * HD;
    const bf16* dobase = dout + (long long)b * Tn * C + h * HD;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q0 = qt * TILE;
    const float sl2 = LOG2E * rsqrtf((float)HD);

    load_tile<HD>(Qs, base, ld, q0, Tn);
    load_tile<HD>(Ds, dobase, C, q0, Tn);
    load_tile<HD>(Ks, base + C, ld, 0, Tn);
    load_tile<HD>(Vs, base + 2 * C, ld, 0, Tn);
    cp_async_commit();

    const int row_g = q0 + warp * 16 + (lane >> 2);
    float Lr[2], Dr[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int q = row_g + r * 8;
        Lr[r] = q < Tn ? lse[(long long)bh * Tn + q] * LOG2E : INFINITY;
        Dr[r] = q < Tn ? dpre[(long long)bh * Tn + q] : 0.f;
    }
    uint32_t qf[HD / 16][4], df[HD / 16][4];
    float dq[HD / 8][4];
    zero<HD / 8>(dq);
    for (int kt = 0; kt <= qt; ++kt) {
        const int buf = kt & 1;
        if (kt + 1 <= qt) {
            load_tile<HD>(Ks + (buf ^ 1) * TILE * Tile<HD>::STRIDE, base + C, ld, (kt + 1) * TILE, Tn);
            load_tile<HD>(Vs + (buf ^ 1) * TILE * Tile<HD>::STRIDE, base + 2 * C, ld, (kt + 1) * TILE, Tn);
        }
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        if (kt == 0) {
            load_a_frags<HD>(qf, Qs, warp * 16);
            load_a_frags<HD>(df, Ds, warp * 16);
        }
        const bf16* Kt = Ks + buf * TILE * Tile<HD>::STRIDE;
        const bf16* Vt = Vs + buf * TILE * Tile<HD>::STRIDE;
        float s[8][4], dp[8][4];
        zero<8>(s);
        zero<8>(dp);
        mma_a_rowsT<HD>(s, qf, Kt);    // S = Q K^T
        mma_a_rowsT<HD>(dp, df, Vt);   // dP = dO V^T
        const bool diag = (kt == qt);
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = kt * TILE + nt * 8 + 2 * (lane & 3) + (e & 1);
                float p = exp2f(s[nt][e] * sl2 - Lr[e >> 1]);
                if (diag && key > row_g + (e >> 1) * 8) p = 0.f;
                s[nt][e] = p * (dp[nt][e] - Dr[e >> 1]);   // dS
            }
        }
        mma_p_rows<HD>(dq, s, Kt);     // dQ += dS K
        __syncthreads();
    }
    const float scale = rsqrtf((float)HD);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int q = row_g + r * 8;
        if (q < Tn) {
            bf16* row = dqkv + ((long long)b * Tn + q) * ld + h * HD;
#pragma unroll
            for (int dt = 0; dt < HD / 8; ++dt) {
                const int col = dt * 8 + 2 * (lane & 3);
                *reinterpret_cast<__nv_bfloat162*>(row + col) =
                    __floats2bfloat162_rn(dq[dt][2 * r] * scale, dq[dt][2 * r + 1] * scale);
            }
        }
    }
}

// D_i = sum_d dO_i,d * O_i,d, one warp per (b, h, i) row group of 4 rows.
template <int HD>
__global__ void flash_bwd_pre_kernel(const bf16* __restrict__ out, const bf16* __restrict__ dout,
                                     float* __restrict__ dpre, int B, int Tn, int H) {
    const long long n = (long long)B * H * Tn;
    const long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= n) return;
    const int i = (int)(g % Tn);
    const int bh = (int)(g / Tn), b = bh / H, h = bh % H;
    const int C = H * HD;
    const long long r = ((long long)b * Tn + i) * C + h * HD;
    float s = 0.f;
#pragma unroll
    for (int d = 0; d < HD; d += 8) {
        const uint4 x = *reinterpret_cast<const uint4*>(out + r + d);
        const uint4 y = *reinterpret_cast<const uint4*>(dout + r + d);
        const __nv_bfloat162* xa = reinterpret_cast<const __nv_bfloat162*>(&x);
        const __nv_bfloat162* ya = reinterpret_cast<const __nv_bfloat162*>(&y);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 fx = __bfloat1622float2(xa[j]), fy = __bfloat1622float2(ya[j]);
            s = fmaf(fx.x, fy.x, fmaf(fx.y, fy.y, s));
        }
    }
    dpre[g] = s;
}

template <int HD>
constexpr int bwd_dkv_smem() {
    return 6 * Tile<HD>::BYTES + 4 * TILE * (int)sizeof(float);
}
template <int HD>
constexpr int bwd_dq_smem() {
    return 6 * Tile<HD>::BYTES;
}

template <int HD>
void fwd_launch(const Ctx& ctx, const bf16* qkv, bf16* out, float* lse, int B, int Tn, int H) {
    dim3 grid(ceil_div(Tn, TILE), B * H);
    flash_fwd_kernel<HD><<<grid, NTHR, 0, ctx.stream>>>(qkv, out, lse, Tn, H);
}

template <int HD>
void bwd_launch(const Ctx& ctx, const bf16* qkv, const bf16* out, const bf16* dout, const float* lse,
                float* dpre, bf16* dqkv, int B, int Tn, int H) {
    static bool configured = false;
    if (!configured) {
        cudaFuncSetAttribute(flash_bwd_dkv_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bwd_dkv_smem<HD>());
        cudaFuncSetAttribute(flash_bwd_dq_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, bwd_dq_smem<HD>());
        configured = true;
    }
    const long long n = (long long)B * H * Tn;
    flash_bwd_pre_kernel<HD><<<(unsigned)ceil_div_ll(n, 256), 256, 0, ctx.stream>>>(out, dout, dpre, B, Tn, H);
    dim3 grid(ceil_div(Tn, TILE), B * H);
    flash_bwd_dkv_kernel<HD><<<grid, NTHR, bwd_dkv_smem<HD>(), ctx.stream>>>(qkv, dout, lse, dpre, dqkv, Tn, H);
    flash_bwd_dq_kernel<HD><<<grid, NTHR, bwd_dq_smem<HD>(), ctx.stream>>>(qkv, dout, lse, dpre, dqkv, Tn, H);
}

}  // namespace

void launch_attention_bwd_pre(const Ctx& ctx, const bf16* out, const bf16* dout, float* dpre, int B, int Tn, int H,
                              int hd) {
    const long long n = (long long)B * H * Tn;
    if (hd == 64)
        flash_bwd_pre_kernel<64><<<(unsigned)ceil_div_ll(n, 256), 256, 0, ctx.stream>>>(out, dout, dpre, B, Tn, H);
    else
        flash_bwd_pre_kernel<32><<<(unsigned)ceil_div_ll(n, 256), 256, 0, ctx.stream>>>(out, dout, dpre, B, Tn, H);
    ++*ctx.launches;
}

void launch_attention_fwd_mma(const Ctx& ctx, const bf16* qkv, bf16* out, float* lse, int B, int Tn, int H,
                              int hd) {
    if (hd == 64) fwd_launch<64>(ctx, qkv, out, lse, B, Tn, H);
    else fwd_launch<32>(ctx, qkv, out, lse, B, Tn, H);
    ++*ctx.launches;
}

void launch_attention_bwd_mma(const Ctx& ctx, const bf16* qkv, const bf16* out, const bf16* dout, const float* lse,
                              float* dpre, bf16* dqkv, int B, int Tn, int H, int hd) {
    if (hd == 64) bwd_launch<64>(ctx, qkv, out, dout, lse, dpre, dqkv, B, Tn, H);
    else bwd_launch<32>(ctx, qkv, out, dout, lse, dpre, dqkv, B, Tn, H);
    *ctx.launches += 3;
}

}  // namespace gpt2
