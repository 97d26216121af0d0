// Causal flash attention forward on the sm_100a tensor cores (tcgen05), head
// width 64, bf16 operands, fp32 softmax and accumulation.
//
// Definition ("GPT-2 from Scratch", "CausalSelfAttention"; "Let's reproduce
// GPT-2 (124M)", "FlashAttention and vocabulary padding"): per (b, h),
// S = q k^T / sqrt(64), keys after the query masked, P = softmax(S), y = P v;
// the softmax is computed online over 128-key tiles with a running row max m
// and row sum l, so no T x T matrix is stored; lse = m + log(l) is kept for
// the backward.
//
// Work item = one (b, h) and 128 queries (one query row per TMEM lane). The
// kernel is persistent: one CTA per SM walks the items, longest causal prefix
// first. Warp 0 loads each item's Q (double-buffered, so the next item's Q
// arrives during the current one) and the K/V tiles of its causal prefix
// through a 3-stage TMA ring; warp 1 issues, from one thread, S_j = Q K_j^T (M=128,
// N=128, K=64) into one of two TMEM S buffers and PV_j = P_j V_j (M=128, N=64,
// K=128; V described as an N-major operand) into one of two TMEM PV buffers;
// warps 2..9 are the softmax warps, two per TMEM lane quarter: each owns 64 of
// the 128 keys of S_j (one 64-key swizzle atom of P) and 32 of the 64 output
// columns. They read S_j from TMEM in two passes (partial row max, exchanged
// with the pair through shared memory; then exp2 / partial row sum / bf16 P
// into the 128-byte-swizzled K-major shared tile), then fold their half of
// PV_{j-1} into the register-resident output row:
// O = O * exp2(m_{j-2} - m_{j-1}) + PV. The pair's row sums meet once at the end.
// Every wait is bounded (2 s) and reports a timeout in the status word.
#include <cudaTypedefs.h>

#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace gpt2 {

namespace {

constexpr int HD = 64;
constexpr int BQ = 128, BKV = 128;
constexpr int KV_STAGES = 3;
constexpr int SM_WARPS = 8;                       // softmax warps: 2 per TMEM lane quarter
constexpr int THREADS = 64 + 32 * SM_WARPS;
constexpr int TILE_BYTES = 128 * HD * 2;          // 16 KB: 128 rows x 128 bytes
constexpr int P_BYTES = BQ * BKV * 2;             // 32 KB: two 64-key swizzle atoms of 16 KB
constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_PV0 = 256, TM_PV1 = 320;
constexpr float LOG2E = 1.4426950408889634f;

struct Ctl {
    uint64_t q_full[2], q_empty[2];
    uint64_t kv_full[KV_STAGES], kv_empty[KV_STAGES];
    uint64_t s_full[2], s_empty[2];
    uint64_t p_full[2];
    uint64_t pv_full[2], pv_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    uint32_t abort;
    float mx[2][2][BQ];                           // [tile parity][column half][row]: partial row max
    float lsum[2][BQ];                            // [column half][row]: partial row sum at the end
};

// smem: Q[2] | K[3] | V[3] | P[2] | ctl
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + 2 * TILE_BYTES;
constexpr int OFF_V = OFF_K + KV_STAGES * TILE_BYTES;
constexpr int OFF_P = OFF_V + KV_STAGES * TILE_BYTES;
constexpr int OFF_CTL = OFF_P + 2 * P_BYTES;
constexpr size_t SMEM_BYTES = OFF_CTL + sizeof(Ctl) + 1024;

__device__ __forceinline__ uint32_t swz128(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

// 2^x with the hardware approximation (ex2.approx; 2^-inf = 0). Its relative
// error (about 2^-22) is far below the bf16 rounding of P and dS.
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void ew_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// max(a, b, c) in one instruction (sm_100 three-input max.f32)
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Max of 32 values in four independent chains of three-input max.
__device__ __forceinline__ float max32(const float* v, float init) {
    float p0 = init, p1 = init, p2 = init, p3 = init;
#pragma unroll
    for (int e = 0; e < 32; e += 8) {
        p0 = max3f(p0, v[e], v[e + 1]);
        p1 = max3f(p1, v[e + 2], v[e + 3]);
        p2 = max3f(p2, v[e + 4], v[e + 5]);
        p3 = max3f(p3, v[e + 6], v[e + 7]);
    }
    return fmaxf(fmaxf(p0, p1), fmaxf(p2, p3));
}

__device__ __forceinline__ uint4 pack8_bf16(const float* v) {
    uint4 q;
    __nv_bfloat162 t0 = __floats2bfloat162_rn(v[0], v[1]);
    __nv_bfloat162 t1 = __floats2bfloat162_rn(v[2], v[3]);
    __nv_bfloat162 t2 = __floats2bfloat162_rn(v[4], v[5]);
    __nv_bfloat162 t3 = __floats2bfloat162_rn(v[6], v[7]);
    q.x = *reinterpret_cast<uint32_t*>(&t0);
    q.y = *reinterpret_cast<uint32_t*>(&t1);
    q.z = *reinterpret_cast<uint32_t*>(&t2);
    q.w = *reinterpret_cast<uint32_t*>(&t3);
    return q;
}

// Work item i of the forward (longest causal prefixes first over the whole
// grid): query tile n_qt - 1 - i / BH of head-sequence i % BH.
struct FwdItem {
    int bh, q0, n_kv;
};
__device__ __forceinline__ FwdItem fwd_item(int i, int BH, int n_qt, int Tn) {
    FwdItem it;
    it.bh = i % BH;
    it.q0 = (n_qt - 1 - i / BH) * BQ;
    it.n_kv = (min(Tn, it.q0 + BQ) + BKV - 1) / BKV;   // key tiles 0 .. n_kv-1
    return it;
}

// Persistent: gridDim.x CTAs (at most one per SM) walk the items
// blockIdx.x, blockIdx.x + gridDim.x, ... Every ring and buffer parity runs on
// counters over all the CTA's tiles, so the loads and S MMAs of the next item
// overlap the softmax and output of the current one.
__global__ void __launch_bounds__(THREADS, 1)
    flash_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, bf16* __restrict__ out, float* __restrict__ lse,
                        int Tn, int H, int BH, unsigned* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctl* ctl = reinterpret_cast<Ctl*>(smem + OFF_CTL);
    volatile uint32_t* abort = &ctl->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_qt = (Tn + BQ - 1) / BQ;
    const int n_items = BH * n_qt;
    const int C = H * HD;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&ctl->q_full[i], 1);
            tc::mbar_init(&ctl->q_empty[i], 1);
            tc::mbar_init(&ctl->s_full[i], 1);
            tc::mbar_init(&ctl->s_empty[i], SM_WARPS);
            tc::mbar_init(&ctl->p_full[i], SM_WARPS);
            tc::mbar_init(&ctl->pv_full[i], 1);
            tc::mbar_init(&ctl->pv_empty[i], SM_WARPS);
        }
        for (int s = 0; s < KV_STAGES; ++s) {
            tc::mbar_init(&ctl->kv_full[s], 1);
            tc::mbar_init(&ctl->kv_empty[s], 1);
        }
        tc::mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        tc::fence_barrier_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(&ctl->tmem_base, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = ctl->tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            // --------------------------------------------------------------- TMA
            tc::tma_prefetch_desc(&tm_qkv);
            uint32_t g = 0;                           // K/V tile counter over all items
            uint32_t ord = 0;                         // item counter (Q buffer ring)
            bool ok = true;
            for (int i = blockIdx.x; i < n_items && ok; i += gridDim.x, ++ord) {
                const FwdItem it = fwd_item(i, BH, n_qt, Tn);
                const int row_base = (it.bh / H) * Tn, h = it.bh % H;
                const int qb = ord & 1;
                if (!tc::mbar_wait(&ctl->q_empty[qb], ((ord >> 1) & 1) ^ 1, abort, status)) break;
                tc::mbar_expect_tx(&ctl->q_full[qb], TILE_BYTES);
                tc::tma_load_2d(smem + OFF_Q + qb * TILE_BYTES, &tm_qkv, h * HD, row_base + it.q0, &ctl->q_full[qb]);
                for (int j = 0; j < it.n_kv; ++j, ++g) {
                    const int s = g % KV_STAGES;
                    const uint32_t ph = (g / KV_STAGES) & 1;
                    if (!tc::mbar_wait(&ctl->kv_empty[s], ph ^ 1, abort, status)) { ok = false; break; }
                    tc::mbar_expect_tx(&ctl->kv_full[s], 2 * TILE_BYTES);
                    tc::tma_load_2d(smem + OFF_K + s * TILE_BYTES, &tm_qkv, C + h * HD, row_base + j * BKV,
                                    &ctl->kv_full[s]);
                    tc::tma_load_2d(smem + OFF_V + s * TILE_BYTES, &tm_qkv, 2 * C + h * HD, row_base + j * BKV,
                                    &ctl->kv_full[s]);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // --------------------------------------------------------------- MMA
            constexpr uint32_t idesc_s = tc::idesc_bf16_f32(BQ, BKV, 0, 0);
            constexpr uint32_t idesc_pv = tc::idesc_bf16_f32(BQ, HD, 0, 1);
            // tile cursor over (item, key tile) in the CTA's order
            struct Cur {
                int i, j, n_kv;
                uint32_t ord;
            };
            auto start = [&](Cur& c, int i, uint32_t ord) {
                c.i = i;
                c.j = 0;
                c.ord = ord;
                c.n_kv = i < n_items ? fwd_item(i, BH, n_qt, Tn).n_kv : 0;
            };
            auto advance = [&](Cur c) {
                Cur n = c;
                if (++n.j == n.n_kv) start(n, c.i + (int)gridDim.x, c.ord + 1);
                return n;
            };
            // S_g = Q K_g^T for the tile at cursor c (global tile index g)
            auto issue_s = [&](const Cur& c, uint32_t g) -> bool {
                const int s = g % KV_STAGES, sb = g & 1, qb = c.ord & 1;
                if (c.j == 0 && !tc::mbar_wait(&ctl->q_full[qb], (c.ord >> 1) & 1, abort, status)) return false;
                if (!tc::mbar_wait(&ctl->kv_full[s], (g / KV_STAGES) & 1, abort, status)) return false;
                if (!tc::mbar_wait(&ctl->s_empty[sb], ((g >> 1) & 1) ^ 1, abort, status)) return false;
                tc::fence_after_sync();
                const uint32_t q_addr = tc::smem_u32(smem + OFF_Q + qb * TILE_BYTES);
                const uint32_t k_addr = tc::smem_u32(smem + OFF_K + s * TILE_BYTES);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk)
                    tc::mma_bf16(tmem + (sb ? TM_S1 : TM_S0), tc::smem_desc_sw128(q_addr + kk * 32, 16, 1024),
                                 tc::smem_desc_sw128(k_addr + kk * 32, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
                tc::mma_commit(&ctl->s_full[sb]);
                if (c.j == c.n_kv - 1) tc::mma_commit(&ctl->q_empty[qb]);   // Q done once this S completes
                return true;
            };
            Cur cur;
            start(cur, blockIdx.x, 0);
            uint32_t g = 0;
            bool ok = cur.i < n_items ? issue_s(cur, 0) : false;
            while (ok && cur.i < n_items) {
                const Cur nxt = advance(cur);
                if (nxt.i < n_items && !issue_s(nxt, g + 1)) break;
                const int s = g % KV_STAGES, pb = g & 1;
                if (!tc::mbar_wait(&ctl->p_full[pb], (g >> 1) & 1, abort, status)) break;
                if (!tc::mbar_wait(&ctl->pv_empty[pb], ((g >> 1) & 1) ^ 1, abort, status)) break;
                tc::fence_after_sync();
                const uint32_t p_addr = tc::smem_u32(smem + OFF_P + pb * P_BYTES);
                const uint32_t v_addr = tc::smem_u32(smem + OFF_V + s * TILE_BYTES);
#pragma unroll
                for (int kk = 0; kk < BKV / 16; ++kk)
                    tc::mma_bf16(tmem + (pb ? TM_PV1 : TM_PV0),
                                 tc::smem_desc_sw128(p_addr + (kk >> 2) * TILE_BYTES + (kk & 3) * 32, 16, 1024),
                                 tc::smem_desc_sw128(v_addr + kk * 2048, TILE_BYTES, 1024), idesc_pv,
                                 kk > 0 ? 1u : 0u);
                tc::mma_commit(&ctl->pv_full[pb]);
                tc::mma_commit(&ctl->kv_empty[s]);
                cur = nxt;
                ++g;
            }
            volatile uint32_t no_abort = 0;
            tc::mma_commit(&ctl->drain);
            tc::mbar_wait(&ctl->drain, 0, &no_abort, status);
        }
    } else {
        // ---------------------------------------------------- softmax / output
        // Warp pair (chalf 0/1) of a lane quarter shares 32 query rows: each warp
        // owns 64 of the 128 keys of an S tile (one swizzle atom of P) and 32 of
        // the 64 output columns. Only the row max is exchanged per tile.
        const int quarter = warp & 3;
        const int chalf = (warp - 2) >> 2;
        const int r = quarter * 32 + lane;            // query row within the tile = TMEM lane
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const float sl2 = LOG2E * 0.125f;             // log2(e) / sqrt(64)
        bool ok = true;
        uint32_t g = 0;                               // tile counter over all items
        float o[32];
        float corr_prev = 1.f;
        auto consume_pv = [&](uint32_t gt) -> bool {
            const int pb = gt & 1;
            uint32_t w = 0;
            if (lane == 0) w = tc::mbar_wait(&ctl->pv_full[pb], (gt >> 1) & 1, abort, status) ? 1u : 0u;
            w = __shfl_sync(0xffffffffu, w, 0);
            if (!w) return false;
            tc::fence_after_sync();
            float pv[32];
            tc::tmem_ld_32x32b_x32(tmem + (pb ? TM_PV1 : TM_PV0) + chalf * 32 + lane_off, pv);
            const f32x2 CP = pk2(corr_prev, corr_prev);
#pragma unroll
            for (int d = 0; d < 32; d += 2)
                upk2(fma2(pk2(o[d], o[d + 1]), CP, pk2(pv[d], pv[d + 1])), o[d], o[d + 1]);
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&ctl->pv_empty[pb]);
            return true;
        };
        // Every softmax warp passes the named barrier n_kv + 2 times per item, also
        // after a failed wait (then without work), so none is left waiting there.
        for (int i = blockIdx.x; i < n_items; i += gridDim.x) {
            const FwdItem it = fwd_item(i, BH, n_qt, Tn);
            const int q0 = it.q0, n_kv = it.n_kv;
            const int q = q0 + r;
#pragma unroll
            for (int d = 0; d < 32; ++d) o[d] = 0.f;
            float m = -INFINITY, l = 0.f;
            corr_prev = 1.f;
            for (int j = 0; j < n_kv; ++j, ++g) {
                const int sb = g & 1;
                uint32_t w = 0;
                if (lane == 0 && ok) w = tc::mbar_wait(&ctl->s_full[sb], (g >> 1) & 1, abort, status) ? 1u : 0u;
                w = __shfl_sync(0xffffffffu, w, 0);
                const uint32_t s_addr = tmem + (sb ? TM_S1 : TM_S0) + chalf * 64 + lane_off;
                const int kbase = j * BKV + chalf * 64;   // first key of this warp's columns
                const bool diag = (j * BKV + BKV > q0);
                // pass 1: partial row max over this warp's 64 keys, exchanged with the pair
                float mx = -INFINITY;
                if (w) {
                    tc::fence_after_sync();
#pragma unroll
                    for (int c = 0; c < 64; c += 32) {
                        float sv[32];
                        tc::tmem_ld_32x32b_x32(s_addr + c, sv);
                        if (diag) {   // keys after the query do not count
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                if (kbase + c + e > q) sv[e] = -INFINITY;
                        }
                        mx = max32(sv, mx);
                    }
                }
                ctl->mx[sb][chalf][r] = mx;
                ew_bar();
                if (!w) { ok = false; continue; }
                mx = fmaxf(mx, ctl->mx[sb][chalf ^ 1][r]);
                const float m_new = fmaxf(m, mx * sl2);
                const float corr = ex2(m - m_new);   // m = -inf at an item's start: 0
                // pass 2: P = exp2(s * sl2 - m_new) as bf16 into this warp's 64-key atom of P
                uint8_t* pt = smem + OFF_P + sb * P_BYTES + chalf * TILE_BYTES;
                // the exponent s * sl2 - m_new and the row sum on packed pairs
                const f32x2 SL = pk2(sl2, sl2), NM = pk2(-m_new, -m_new);
                f32x2 RS = pk2(0.f, 0.f);
#pragma unroll
                for (int c = 0; c < 64; c += 32) {
                    float sv[32];
                    tc::tmem_ld_32x32b_x32(s_addr + c, sv);
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        float t0, t1;
                        upk2(fma2(pk2(sv[e], sv[e + 1]), SL, NM), t0, t1);
                        sv[e] = ex2(t0);
                        sv[e + 1] = ex2(t1);
                    }
                    if (diag) {
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (kbase + c + e > q) sv[e] = 0.f;
                    }
#pragma unroll
                    for (int e = 0; e < 32; e += 2) RS = add2(RS, pk2(sv[e], sv[e + 1]));
#pragma unroll
                    for (int gg = 0; gg < 4; ++gg)
                        *reinterpret_cast<uint4*>(pt + swz128(r, (c >> 3) + gg)) = pack8_bf16(sv + 8 * gg);
                }
                float rs0, rs1;
                upk2(RS, rs0, rs1);
                const float rs = rs0 + rs1;
                l = l * corr + rs;
                m = m_new;
                tc::fence_proxy_async_smem();      // P visible to the tensor core
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) {
                    tc::mbar_arrive(&ctl->p_full[sb]);
                    tc::mbar_arrive(&ctl->s_empty[sb]);
                }
                if (j > 0 && !consume_pv(g - 1)) { ok = false; continue; }
                corr_prev = corr;
            }
            if (ok && n_kv > 0) ok = consume_pv(g - 1);
            // row sum of both halves
            ctl->lsum[chalf][r] = l;
            ew_bar();
            const float l_tot = l + ctl->lsum[chalf ^ 1][r];
            // out rows: O / l, staged in the first 64-key atom of P buffer 0 (every PV MMA of
            // this item has completed; only these warps write P, and only after this store)
            uint8_t* stage = smem + OFF_P;
            if (ok) {
                const float inv = 1.f / l_tot;
#pragma unroll
                for (int gg = 0; gg < 4; ++gg) {
                    float t[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) t[e] = o[8 * gg + e] * inv;
                    *reinterpret_cast<uint4*>(stage + swz128(r, chalf * 4 + gg)) = pack8_bf16(t);
                }
                if (chalf == 0 && q < Tn) lse[(long long)it.bh * Tn + q] = (m + log2f(l_tot)) / LOG2E;
            }
            ew_bar();
            if (ok && chalf == 0) {
                const int b = it.bh / H, h = it.bh % H;
                const int lrow = lane >> 3, lseg = lane & 7;
#pragma unroll
                for (int st = 0; st < 8; ++st) {
                    const int rr = quarter * 32 + st * 4 + lrow;
                    if (q0 + rr < Tn)
                        *reinterpret_cast<uint4*>(out + ((long long)b * Tn + q0 + rr) * C + h * HD + lseg * 8) =
                            *reinterpret_cast<const uint4*>(stage + swz128(rr, lseg));
                }
                __syncwarp();
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

// ============================================================================
// Backward. D = rowsum(dO * O) comes from the pre-pass kernel. With
// P = exp(S - lse) recomputed from the saved lse:
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),
//   dK = dS^T Q / sqrt(64),  dQ = dS K / sqrt(64).
// dK/dV kernel: one CTA per (b, h, 128-key tile); it walks the 64-query tiles
// at or after the key tile. K and V are copied once into TMEM as packed bf16
// A operands, so the N=64 MMAs read only their B operand from shared memory
// (with both operands there they are limited by shared-memory bandwidth).
// S^T = K Q^T and dP^T = V dO^T (M=128 keys, N=64 queries) go to
// double-buffered TMEM so the tensor core computes tile i+1 while 8 warps turn
// tile i into P^T and dS^T, written back as packed bf16 over the S^T / dP^T
// columns they came from; dV += P^T dO and dK += dS^T Q (A from TMEM; dO and Q
// as N-major shared operands) accumulate in TMEM. dQ kernel: one CTA per (b, h, 128-query tile) over the 64-key tiles at
// or before it: S = Q K^T, dP = dO V^T, dS, then dQ += dS K in TMEM.
// ============================================================================
constexpr int BW_EW_WARPS = 8;                     // 2 warps per TMEM lane quarter, 32 columns each
constexpr int BW_THREADS = 64 + 32 * BW_EW_WARPS;
constexpr int T64_BYTES = 64 * HD * 2;      // 8 KB: 64 rows x 128 bytes
constexpr int T128_BYTES = 128 * HD * 2;    // 16 KB

// Write one 64-column bf16 result row (128 bytes) per thread of a 4-warp group
// through a swizzled 128-row staging tile, then copy whole rows to global
// memory: dst(row) = base + row * ld (elements), rows >= n_rows skipped.
// If csum is non-null, the warp also writes the column sums of its 32 rows
// (rows at or beyond n_rows excluded) of the stored bf16 values as 64 floats
// at csum; a warp whose rows all lie beyond n_rows writes nothing.
__device__ __forceinline__ void store_rows_64(uint8_t* stage, int r, const float* v, float scale, bf16* base,
                                              long long ld, int n_rows, float* csum) {
    const int lane = threadIdx.x & 31, quarter = (threadIdx.x >> 5) & 3;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        float t[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) t[e] = v[8 * c + e] * scale;
        *reinterpret_cast<uint4*>(stage + swz128(r, c)) = pack8_bf16(t);
    }
    __syncwarp();
    const int lrow = lane >> 3, lseg = lane & 7;
#pragma unroll
    for (int st = 0; st < 8; ++st) {
        const int rr = quarter * 32 + st * 4 + lrow;
        if (rr < n_rows)
            *reinterpret_cast<uint4*>(base + (long long)rr * ld + lseg * 8) =
                *reinterpret_cast<const uint4*>(stage + swz128(rr, lseg));
    }
    if (csum && quarter * 32 < n_rows) {   // lane = columns 2 lane, 2 lane + 1
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int rr = quarter * 32 + i;
            if (rr < n_rows) {
                const uint32_t w2 = *reinterpret_cast<const uint32_t*>(stage + swz128(rr, lane >> 2) + (lane & 3) * 4);
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w2));
                s0 += f.x;
                s1 += f.y;
            }
        }
        *reinterpret_cast<float2*>(csum + 2 * lane) = make_float2(s0, s1);
    }
    __syncwarp();
}

constexpr int DKV_STAGES = 6;   // Q/dO ring deep enough to cover a ~1.3 us tile load
struct CtlDkv {
    uint64_t kv_full;
    uint64_t q_full[DKV_STAGES], q_empty[DKV_STAGES];
    uint64_t st_full[2], st_empty[2];
    uint64_t ew_done[2];
    uint64_t kv_tmem;                            // K and V copied into TMEM (A operands)
    uint64_t acc_done;
    uint64_t drain;
    uint32_t tmem_base;
    uint32_t abort;
    alignas(16) float lse2[2][64];   // negated, log2 units (read as float2 pairs)
    alignas(16) float dd[2][64];     // negated D
};
// smem: K | V | (Q | dO) stages | output staging | ctl
constexpr int DKV_OFF_K = 0;
constexpr int DKV_OFF_V = DKV_OFF_K + T128_BYTES;
constexpr int DKV_OFF_Q = DKV_OFF_V + T128_BYTES;
constexpr int DKV_STAGE_BYTES = 2 * T64_BYTES;                  // Q tile + dO tile
constexpr int DKV_OFF_STAGE = DKV_OFF_Q + DKV_STAGES * DKV_STAGE_BYTES;   // dK / dV output staging
constexpr int DKV_OFF_CTL = DKV_OFF_STAGE + T128_BYTES;
constexpr size_t DKV_SMEM = DKV_OFF_CTL + sizeof(CtlDkv) + 1024;
// TMEM columns
// TMEM columns: S^T and dP^T (fp32, double-buffered; after the element-wise step
// the first 16 columns of each 32-column half hold that half's P^T / dS^T as
// packed bf16, the A operand of the dV / dK MMAs), the dV and dK accumulators,
// and K and V as packed bf16 A operands of the S^T and dP^T MMAs.
constexpr uint32_t DKV_ST = 0, DKV_DPT = 128, DKV_DV = 256, DKV_DK = 320, DKV_KT = 384, DKV_VT = 416;

__global__ void __launch_bounds__(BW_THREADS, 1)
    flash_bwd_dkv_tc_kernel(const __grid_constant__ CUtensorMap tm_kv, const __grid_constant__ CUtensorMap tm_q,
                            const __grid_constant__ CUtensorMap tm_do, const float* __restrict__ lse,
                            const float* __restrict__ dpre, bf16* __restrict__ dqkv, int Tn, int H,
                            float* __restrict__ colsum_part, unsigned* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    CtlDkv* ctl = reinterpret_cast<CtlDkv*>(smem + DKV_OFF_CTL);
    volatile uint32_t* abort = &ctl->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // grid (B H, key tiles): key tile 0 sees the most queries and is dispatched first
    const int kt = blockIdx.y;
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const int C = H * HD;
    const int k0 = kt * 128;
    const int n_q64 = (Tn + 63) / 64;
    const int it0 = k0 / 64;                            // first 64-query tile that sees these keys
    const int n_it = n_q64 - it0;
    const int row_base = b * Tn;

    if (threadIdx.x == 0) {
        tc::mbar_init(&ctl->kv_full, 1);
        for (int s = 0; s < DKV_STAGES; ++s) {
            tc::mbar_init(&ctl->q_full[s], 1);
            tc::mbar_init(&ctl->q_empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&ctl->st_full[i], 1);
            tc::mbar_init(&ctl->st_empty[i], BW_EW_WARPS);
            tc::mbar_init(&ctl->ew_done[i], BW_EW_WARPS);
        }
        tc::mbar_init(&ctl->kv_tmem, BW_EW_WARPS);
        tc::mbar_init(&ctl->acc_done, 1);
        tc::mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        tc::fence_barrier_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(&ctl->tmem_base, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = ctl->tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            tc::tma_prefetch_desc(&tm_kv);
            tc::tma_prefetch_desc(&tm_q);
            tc::tma_prefetch_desc(&tm_do);
            tc::mbar_expect_tx(&ctl->kv_full, 2 * T128_BYTES);
            tc::tma_load_2d(smem + DKV_OFF_K, &tm_kv, C + h * HD, row_base + k0, &ctl->kv_full);
            tc::tma_load_2d(smem + DKV_OFF_V, &tm_kv, 2 * C + h * HD, row_base + k0, &ctl->kv_full);
            for (int it = 0; it < n_it; ++it) {
                const int s = it % DKV_STAGES;
                if (!tc::mbar_wait(&ctl->q_empty[s], ((it / DKV_STAGES) & 1) ^ 1, abort, status)) break;
                const int q0 = (it0 + it) * 64;
                uint8_t* st = smem + DKV_OFF_Q + s * DKV_STAGE_BYTES;
                tc::mbar_expect_tx(&ctl->q_full[s], 2 * T64_BYTES);
                tc::tma_load_2d(st, &tm_q, h * HD, row_base + q0, &ctl->q_full[s]);
                tc::tma_load_2d(st + T64_BYTES, &tm_do, h * HD, row_base + q0, &ctl->q_full[s]);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc_st = tc::idesc_bf16_f32(128, 64, 0, 0);   // K Q^T, V dO^T
            constexpr uint32_t idesc_acc = tc::idesc_bf16_f32(128, 64, 0, 1);  // P^T dO, dS^T Q
            bool ok = tc::mbar_wait(&ctl->kv_tmem, 0, abort, status);
            auto accumulate = [&](int it) -> bool {   // dV += P^T dO, dK += dS^T Q for tile it
                const int r = it & 1, s = it % DKV_STAGES;
                if (!tc::mbar_wait(&ctl->ew_done[r], (it >> 1) & 1, abort, status)) return false;
                tc::fence_after_sync();
                const uint32_t q_addr = tc::smem_u32(smem + DKV_OFF_Q + s * DKV_STAGE_BYTES);
                const uint32_t do_addr = q_addr + T64_BYTES;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {   // K = 64 queries: 16 per MMA, 8 packed columns
                    const uint32_t acc = (it > 0 || kk > 0) ? 1u : 0u;
                    const uint32_t col = r * 64 + (kk >> 1) * 32 + (kk & 1) * 8;
                    tc::mma_bf16_ts(tmem + DKV_DV, tmem + DKV_ST + col,
                                    tc::smem_desc_sw128(do_addr + kk * 2048, T64_BYTES, 1024), idesc_acc, acc);
                    tc::mma_bf16_ts(tmem + DKV_DK, tmem + DKV_DPT + col,
                                    tc::smem_desc_sw128(q_addr + kk * 2048, T64_BYTES, 1024), idesc_acc, acc);
                }
                tc::mma_commit(&ctl->q_empty[s]);
                return true;
            };
            for (int it = 0; it < n_it && ok; ++it) {
                const int r = it & 1, s = it % DKV_STAGES;
                if (!tc::mbar_wait(&ctl->q_full[s], (it / DKV_STAGES) & 1, abort, status)) break;
                if (!tc::mbar_wait(&ctl->st_empty[r], ((it >> 1) & 1) ^ 1, abort, status)) break;
                tc::fence_after_sync();
                const uint32_t q_addr = tc::smem_u32(smem + DKV_OFF_Q + s * DKV_STAGE_BYTES);
                const uint32_t do_addr = q_addr + T64_BYTES;
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    tc::mma_bf16_ts(tmem + DKV_ST + r * 64, tmem + DKV_KT + kk * 8,
                                    tc::smem_desc_sw128(q_addr + kk * 32, 16, 1024), idesc_st, kk > 0 ? 1u : 0u);
                    tc::mma_bf16_ts(tmem + DKV_DPT + r * 64, tmem + DKV_VT + kk * 8,
                                    tc::smem_desc_sw128(do_addr + kk * 32, 16, 1024), idesc_st, kk > 0 ? 1u : 0u);
                }
                tc::mma_commit(&ctl->st_full[r]);
                if (it > 0 && !accumulate(it - 1)) { ok = false; break; }
            }
            if (ok && n_it > 0) ok = accumulate(n_it - 1);
            tc::mma_commit(&ctl->acc_done);
            volatile uint32_t no_abort = 0;
            tc::mma_commit(&ctl->drain);
            tc::mbar_wait(&ctl->drain, 0, &no_abort, status);
        }
    } else {
        // ------------------------------------------- P^T, dS^T (thread = key row)
        const int quarter = warp & 3;
        const int chalf = (warp - 2) >> 2;              // query columns [32 chalf, 32 chalf + 32)
        const int r = quarter * 32 + lane;              // key row in the tile = TMEM lane
        const int key = k0 + r;
        const int et = threadIdx.x - 64;                // 0..255 within the element-wise warps
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const float sl2 = LOG2E * 0.125f;
        // per-query lse (log2 units) and D of the next tile, one value per thread
        // stored negated, the form the packed exponent and dS arithmetic take
        auto fetch = [&](int it) -> float {
            const int q = (it0 + it) * 64 + (et & 63);
            if (et < 64) return q < Tn ? -lse[(long long)bh * Tn + q] * LOG2E : -INFINITY;
            if (et < 128) return q < Tn ? -dpre[(long long)bh * Tn + q] : 0.f;
            return 0.f;
        };
        // two tiles of lookahead: a global load's latency exceeds one tile's work
        float nxt = n_it > 0 ? fetch(0) : 0.f;
        float nxt2 = n_it > 1 ? fetch(1) : 0.f;
        bool ok = true;
        {
            // K and V rows into TMEM as the packed bf16 A operands of the S^T and dP^T MMAs:
            // this thread's key row, head columns [32 chalf, 32 chalf + 32) = 16 columns
            uint32_t w = 0;
            if (lane == 0) w = tc::mbar_wait(&ctl->kv_full, 0, abort, status) ? 1u : 0u;
            w = __shfl_sync(0xffffffffu, w, 0);
            if (w) {
                uint32_t kw[16], vw[16];
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const uint4 kq = *reinterpret_cast<const uint4*>(smem + DKV_OFF_K + swz128(r, chalf * 4 + g));
                    const uint4 vq = *reinterpret_cast<const uint4*>(smem + DKV_OFF_V + swz128(r, chalf * 4 + g));
                    kw[4 * g] = kq.x; kw[4 * g + 1] = kq.y; kw[4 * g + 2] = kq.z; kw[4 * g + 3] = kq.w;
                    vw[4 * g] = vq.x; vw[4 * g + 1] = vq.y; vw[4 * g + 2] = vq.z; vw[4 * g + 3] = vq.w;
                }
                tc::tmem_st_32x32b_x16(tmem + DKV_KT + chalf * 16 + lane_off, kw);
                tc::tmem_st_32x32b_x16(tmem + DKV_VT + chalf * 16 + lane_off, vw);
                tc::tmem_wait_st();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&ctl->kv_tmem);
            } else {
                ok = false;
            }
        }
        for (int it = 0; it < n_it; ++it) {
            const int rb = it & 1;
            const int q0 = (it0 + it) * 64;
            if (et < 64) ctl->lse2[rb][et] = nxt;
            else if (et < 128) ctl->dd[rb][et - 64] = nxt;
            ew_bar();
            nxt = nxt2;
            if (it + 2 < n_it) nxt2 = fetch(it + 2);
            uint32_t w = 0;
            // st_full also means every earlier MMA is done, among them the dV/dK MMAs that
            // read this buffer's P^T / dS^T two tiles ago
            if (lane == 0 && ok) w = tc::mbar_wait(&ctl->st_full[rb], (it >> 1) & 1, abort, status) ? 1u : 0u;
            w = __shfl_sync(0xffffffffu, w, 0);
            // after a failed wait keep looping without work, so that every
            // element-wise warp reaches the named barrier equally often
            if (!w) { ok = false; continue; }
            tc::fence_after_sync();
            const bool diag = (q0 < k0 + 128);          // some queries of the tile precede some keys
            float sv[32], dp[32];
            tc::tmem_ld2_32x32b_x32(tmem + DKV_ST + rb * 64 + chalf * 32 + lane_off,
                                    tmem + DKV_DPT + rb * 64 + chalf * 32 + lane_off, sv, dp);
            // P^T = 2^(s sl2 - lse2), dS^T = P^T (dP^T - D) on packed pairs of queries
            const f32x2 SL = pk2(sl2, sl2);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
                const int qi = chalf * 32 + e;
                const float2 nl = *reinterpret_cast<const float2*>(&ctl->lse2[rb][qi]);
                const float2 nd = *reinterpret_cast<const float2*>(&ctl->dd[rb][qi]);
                float t0, t1;
                upk2(fma2(pk2(sv[e], sv[e + 1]), SL, pk2(nl.x, nl.y)), t0, t1);
                sv[e] = ex2(t0);
                sv[e + 1] = ex2(t1);
                if (diag) {   // queries before this key
                    if (key > q0 + qi) sv[e] = 0.f;
                    if (key > q0 + qi + 1) sv[e + 1] = 0.f;
                }
                upk2(mul2(pk2(sv[e], sv[e + 1]), add2(pk2(dp[e], dp[e + 1]), pk2(nd.x, nd.y))), dp[e], dp[e + 1]);
            }
            // P^T and dS^T as packed bf16 over the first 16 columns of this warp's S^T / dP^T half
            uint32_t pw[16], dw[16];
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                const uint4 a = pack8_bf16(sv + 8 * g), d = pack8_bf16(dp + 8 * g);
                pw[4 * g] = a.x; pw[4 * g + 1] = a.y; pw[4 * g + 2] = a.z; pw[4 * g + 3] = a.w;
                dw[4 * g] = d.x; dw[4 * g + 1] = d.y; dw[4 * g + 2] = d.z; dw[4 * g + 3] = d.w;
            }
            tc::tmem_st_32x32b_x16(tmem + DKV_ST + rb * 64 + chalf * 32 + lane_off, pw);
            tc::tmem_st_32x32b_x16(tmem + DKV_DPT + rb * 64 + chalf * 32 + lane_off, dw);
            tc::tmem_wait_st();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                tc::mbar_arrive(&ctl->st_empty[rb]);
                tc::mbar_arrive(&ctl->ew_done[rb]);
            }
        }
        if (ok && chalf == 0) {
            uint32_t w = 0;
            if (lane == 0) w = tc::mbar_wait(&ctl->acc_done, 0, abort, status) ? 1u : 0u;
            w = __shfl_sync(0xffffffffu, w, 0);
            if (w) {
                tc::fence_after_sync();
                float v[64];
                tc::tmem_ld_32x32b_x64(tmem + DKV_DK + lane_off, v);
                bf16* kbase = dqkv + ((long long)row_base + k0) * 3 * C + C + h * HD;
                uint8_t* stage = smem + DKV_OFF_STAGE;
                // column sums (the c_attn bias gradient) of this warp's 32-row group
                float* cs = colsum_part ? colsum_part + ((long long)b * ((Tn + 31) / 32) + kt * 4 + quarter) * 3 * C
                                        : nullptr;
                store_rows_64(stage, r, v, 0.125f, kbase, 3LL * C, Tn - k0, cs ? cs + C + h * HD : nullptr);
                tc::tmem_ld_32x32b_x64(tmem + DKV_DV + lane_off, v);
                store_rows_64(stage, r, v, 1.0f, kbase + C, 3LL * C, Tn - k0, cs ? cs + 2 * C + h * HD : nullptr);
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

constexpr int DQ_STAGES = 6;    // K/V ring, likewise
struct CtlDq {
    uint64_t q_full;
    uint64_t kv_full[DQ_STAGES], kv_empty[DQ_STAGES];
    uint64_t s_full[2], s_empty[2];
    uint64_t ds_full[2], ds_free[2];
    uint64_t acc_done;
    uint64_t drain;
    uint32_t tmem_base;
    uint32_t abort;
};
// smem: Q | dO | (K | V) stages | dS[2] | ctl
constexpr int DQ_OFF_Q = 0;
constexpr int DQ_OFF_DO = DQ_OFF_Q + T128_BYTES;
constexpr int DQ_OFF_KV = DQ_OFF_DO + T128_BYTES;
constexpr int DQ_STAGE_BYTES = 2 * T64_BYTES;
constexpr int DQ_OFF_DS = DQ_OFF_KV + DQ_STAGES * DQ_STAGE_BYTES;
constexpr int DQ_OFF_CTL = DQ_OFF_DS + 2 * T128_BYTES;   // 128 queries x 64 keys bf16 = 16 KB each
constexpr size_t DQ_SMEM = DQ_OFF_CTL + sizeof(CtlDq) + 1024;
constexpr uint32_t DQ_S = 0, DQ_DP = 128, DQ_DQ = 256;

__global__ void __launch_bounds__(BW_THREADS, 1)
    flash_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q128, const __grid_constant__ CUtensorMap tm_kv64,
                           const __grid_constant__ CUtensorMap tm_do128, const float* __restrict__ lse,
                           const float* __restrict__ dpre, bf16* __restrict__ dqkv, int Tn, int H,
                           float* __restrict__ colsum_part, unsigned* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    CtlDq* ctl = reinterpret_cast<CtlDq*>(smem + DQ_OFF_CTL);
    volatile uint32_t* abort = &ctl->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // grid (B H, query tiles): the last query tile sees the most keys and is dispatched first
    const int n_qt = gridDim.y;
    const int qt = n_qt - 1 - blockIdx.y;
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const int C = H * HD;
    const int q0 = qt * 128;
    const int n_k64 = (min(Tn, q0 + 128) + 63) / 64;    // key tiles that some query of the tile sees
    const int row_base = b * Tn;

    if (threadIdx.x == 0) {
        tc::mbar_init(&ctl->q_full, 1);
        for (int s = 0; s < DQ_STAGES; ++s) {
            tc::mbar_init(&ctl->kv_full[s], 1);
            tc::mbar_init(&ctl->kv_empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&ctl->s_full[i], 1);
            tc::mbar_init(&ctl->s_empty[i], BW_EW_WARPS);
            tc::mbar_init(&ctl->ds_full[i], BW_EW_WARPS);
            tc::mbar_init(&ctl->ds_free[i], 1);
        }
        tc::mbar_init(&ctl->acc_done, 1);
        tc::mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        tc::fence_barrier_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(&ctl->tmem_base, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = ctl->tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            tc::tma_prefetch_desc(&tm_q128);
            tc::tma_prefetch_desc(&tm_kv64);
            tc::tma_prefetch_desc(&tm_do128);
            tc::mbar_expect_tx(&ctl->q_full, 2 * T128_BYTES);
            tc::tma_load_2d(smem + DQ_OFF_Q, &tm_q128, h * HD, row_base + q0, &ctl->q_full);
            tc::tma_load_2d(smem + DQ_OFF_DO, &tm_do128, h * HD, row_base + q0, &ctl->q_full);
            for (int j = 0; j < n_k64; ++j) {
                const int s = j % DQ_STAGES;
                if (!tc::mbar_wait(&ctl->kv_empty[s], ((j / DQ_STAGES) & 1) ^ 1, abort, status)) break;
                uint8_t* st = smem + DQ_OFF_KV + s * DQ_STAGE_BYTES;
                tc::mbar_expect_tx(&ctl->kv_full[s], 2 * T64_BYTES);
                tc::tma_load_2d(st, &tm_kv64, C + h * HD, row_base + j * 64, &ctl->kv_full[s]);
                tc::tma_load_2d(st + T64_BYTES, &tm_kv64, 2 * C + h * HD, row_base + j * 64, &ctl->kv_full[s]);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc_s = tc::idesc_bf16_f32(128, 64, 0, 0);    // Q K^T, dO V^T
            constexpr uint32_t idesc_dq = tc::idesc_bf16_f32(128, 64, 0, 1);   // dS K
            const uint32_t q_addr = tc::smem_u32(smem + DQ_OFF_Q), do_addr = tc::smem_u32(smem + DQ_OFF_DO);
            bool ok = tc::mbar_wait(&ctl->q_full, 0, abort, status);
            auto accumulate = [&](int j) -> bool {   // dQ += dS K for key tile j
                const int r = j & 1, s = j % DQ_STAGES;
                if (!tc::mbar_wait(&ctl->ds_full[r], (j >> 1) & 1, abort, status)) return false;
                tc::fence_after_sync();
                const uint32_t k_addr = tc::smem_u32(smem + DQ_OFF_KV + s * DQ_STAGE_BYTES);
                const uint32_t ds = tc::smem_u32(smem + DQ_OFF_DS + r * T128_BYTES);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)   // K = 64 keys
                    tc::mma_bf16(tmem + DQ_DQ, tc::smem_desc_sw128(ds + kk * 32, 16, 1024),
                                 tc::smem_desc_sw128(k_addr + kk * 2048, T64_BYTES, 1024), idesc_dq,
                                 (j > 0 || kk > 0) ? 1u : 0u);
                tc::mma_commit(&ctl->ds_free[r]);
                tc::mma_commit(&ctl->kv_empty[s]);
                return true;
            };
            for (int j = 0; j < n_k64 && ok; ++j) {
                const int r = j & 1, s = j % DQ_STAGES;
                if (!tc::mbar_wait(&ctl->kv_full[s], (j / DQ_STAGES) & 1, abort, status)) break;
                if (!tc::mbar_wait(&ctl->s_empty[r], ((j >> 1) & 1) ^ 1, abort, status)) break;
                tc::fence_after_sync();
                const uint32_t k_addr = tc::smem_u32(smem + DQ_OFF_KV + s * DQ_STAGE_BYTES);
                const uint32_t v_addr = k_addr + T64_BYTES;
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    tc::mma_bf16(tmem + DQ_S + r * 64, tc::smem_desc_sw128(q_addr + kk * 32, 16, 1024),
                                 tc::smem_desc_sw128(k_addr + kk * 32, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
                    tc::mma_bf16(tmem + DQ_DP + r * 64, tc::smem_desc_sw128(do_addr + kk * 32, 16, 1024),
                                 tc::smem_desc_sw128(v_addr + kk * 32, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
                }
                tc::mma_commit(&ctl->s_full[r]);
                if (j > 0 && !accumulate(j - 1)) { ok = false; break; }
            }
            if (ok && n_k64 > 0) ok = accumulate(n_k64 - 1);
            tc::mma_commit(&ctl->acc_done);
            volatile uint32_t no_abort = 0;
            tc::mma_commit(&ctl->drain);
            tc::mbar_wait(&ctl->drain, 0, &no_abort, status);
        }
    } else {
        // --------------------------------------------------- dS (thread = query row)
        const int quarter = warp & 3;
        const int chalf = (warp - 2) >> 2;              // key columns [32 chalf, 32 chalf + 32)
        const int r = quarter * 32 + lane;
        const int q = q0 + r;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const float sl2 = LOG2E * 0.125f;
        const float L2 = q < Tn ? lse[(long long)bh * Tn + q] * LOG2E : INFINITY;
        const float Dv = q < Tn ? dpre[(long long)bh * Tn + q] : 0.f;
        bool ok = true;
        for (int j = 0; j < n_k64; ++j) {
            const int rb = j & 1;
            uint32_t w = 0;
            if (lane == 0) {
                w = tc::mbar_wait(&ctl->s_full[rb], (j >> 1) & 1, abort, status) ? 1u : 0u;
                if (w) w = tc::mbar_wait(&ctl->ds_free[rb], ((j >> 1) & 1) ^ 1, abort, status) ? 1u : 0u;
            }
            w = __shfl_sync(0xffffffffu, w, 0);
            if (!w) { ok = false; break; }
            tc::fence_after_sync();
            const bool diag = (j * 64 + 64 > q0);
            uint8_t* ds = smem + DQ_OFF_DS + rb * T128_BYTES;
            float sv[32], dp[32];
            tc::tmem_ld2_32x32b_x32(tmem + DQ_S + rb * 64 + chalf * 32 + lane_off,
                                    tmem + DQ_DP + rb * 64 + chalf * 32 + lane_off, sv, dp);
            // dS = 2^(s sl2 - lse2) (dP - D) on packed pairs of keys
            const f32x2 SL = pk2(sl2, sl2), NL = pk2(-L2, -L2), ND = pk2(-Dv, -Dv);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
                float t0, t1;
                upk2(fma2(pk2(sv[e], sv[e + 1]), SL, NL), t0, t1);
                float p0 = ex2(t0), p1 = ex2(t1);
                if (diag) {   // keys after this query
                    if (j * 64 + chalf * 32 + e > q) p0 = 0.f;
                    if (j * 64 + chalf * 32 + e + 1 > q) p1 = 0.f;
                }
                upk2(mul2(pk2(p0, p1), add2(pk2(dp[e], dp[e + 1]), ND)), dp[e], dp[e + 1]);
            }
#pragma unroll
            for (int g = 0; g < 4; ++g)
                *reinterpret_cast<uint4*>(ds + swz128(r, chalf * 4 + g)) = pack8_bf16(dp + 8 * g);
            tc::fence_proxy_async_smem();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                tc::mbar_arrive(&ctl->s_empty[rb]);
                tc::mbar_arrive(&ctl->ds_full[rb]);
            }
        }
        if (ok && chalf == 0) {
            uint32_t w = 0;
            if (lane == 0) w = tc::mbar_wait(&ctl->acc_done, 0, abort, status) ? 1u : 0u;
            w = __shfl_sync(0xffffffffu, w, 0);
            if (w) {
                tc::fence_after_sync();
                float v[64];
                tc::tmem_ld_32x32b_x64(tmem + DQ_DQ + lane_off, v);
                bf16* qbase = dqkv + ((long long)row_base + q0) * 3 * C + h * HD;
                float* cs = colsum_part ? colsum_part + ((long long)b * ((Tn + 31) / 32) + qt * 4 + quarter) * 3 * C
                                        : nullptr;
                store_rows_64(smem + DQ_OFF_DS, r, v, 0.125f, qbase, 3LL * C, Tn - q0, cs ? cs + h * HD : nullptr);
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn_attn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

}  // namespace

bool attention_tc_supported(int hd) { return hd == HD && encode_fn_attn() != nullptr; }

bool launch_attention_fwd_tc(const Ctx& ctx, const bf16* qkv, bf16* out, float* lse, int B, int Tn, int H) {
    auto fn = encode_fn_attn();
    if (!fn) return false;
    const long long C = (long long)H * HD;
    CUtensorMap m;
    cuuint64_t dims[2] = {(cuuint64_t)(3 * C), (cuuint64_t)B * Tn};
    cuuint64_t strides[1] = {(cuuint64_t)(3 * C) * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<bf16*>(qkv), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    static bool configured = false;
    if (!configured) {
        cudaFuncSetAttribute(flash_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
        configured = true;
    }
    const int n_items = B * H * ceil_div(Tn, BQ);
    const int grid = min(n_items, ctx.num_sms > 0 ? ctx.num_sms : 148);
    flash_fwd_tc_kernel<<<grid, THREADS, SMEM_BYTES, ctx.stream>>>(m, out, lse, Tn, H, B * H, ctx.status);
    ++*ctx.launches;
    return true;
}

bool launch_attention_bwd_tc(const Ctx& ctx, const bf16* qkv, const bf16* out, const bf16* dout, const float* lse,
                             float* dpre, bf16* dqkv, int B, int Tn, int H, float* colsum_part) {
    auto fn = encode_fn_attn();
    if (!fn) return false;
    const long long C = (long long)H * HD;
    auto make = [&](CUtensorMap* m, const bf16* base, long long cols, int box_rows) {
        cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)B * Tn};
        cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
        cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
        cuuint32_t estr[2] = {1, 1};
        return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<bf16*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    };
    CUtensorMap qkv128, qkv64, do64, do128;
    if (!make(&qkv128, qkv, 3 * C, 128) || !make(&qkv64, qkv, 3 * C, 64) || !make(&do64, dout, C, 64) ||
        !make(&do128, dout, C, 128))
        return false;
    static bool configured = false;
    if (!configured) {
        cudaFuncSetAttribute(flash_bwd_dkv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)DKV_SMEM);
        cudaFuncSetAttribute(flash_bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)DQ_SMEM);
        configured = true;
    }
    launch_attention_bwd_pre(ctx, out, dout, dpre, B, Tn, H, HD);
    const dim3 grid(B * H, ceil_div(Tn, 128));
    flash_bwd_dkv_tc_kernel<<<grid, BW_THREADS, DKV_SMEM, ctx.stream>>>(qkv128, qkv64, do64, lse, dpre, dqkv, Tn, H,
                                                                         colsum_part, ctx.status);
    flash_bwd_dq_tc_kernel<<<grid, BW_THREADS, DQ_SMEM, ctx.stream>>>(qkv128, qkv64, do128, lse, dpre, dqkv, Tn, H,
                                                                       colsum_part, ctx.status);
    *ctx.launches += 2;
    return true;
}

}  // namespace gpt2
