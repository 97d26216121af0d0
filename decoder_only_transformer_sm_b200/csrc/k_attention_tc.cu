// Causal flash attention forward and backward on the sm_100a tensor cores
// (tcgen05), head width 64, bf16 operands, fp32 softmax and accumulation. The
// backward is described above its kernel, further down.
//
// Definition ("GPT-2 from Scratch", "CausalSelfAttention"; "Let's reproduce
// GPT-2 (124M)", "FlashAttention and vocabulary padding"): per (b, h),
// S = q k^T / sqrt(64), keys after the query masked, P = softmax(S), y = P v;
// the softmax is computed online over 128-key tiles with a running row max m
// and row sum l, so no T x T matrix is stored; lse = m + log(l) is kept for
// the backward.
//
// Work item = one (b, h) and a pair of consecutive 128-query tiles (2p, 2p+1),
// one per softmax warpgroup ("group"); both walk the same key tiles, so each K/V
// tile is loaded once for the pair. The kernel is persistent: one CTA per SM
// walks the items, longest causal prefixes first, dealt to the CTAs round by
// round in alternating direction. Warp 0 loads an item's two Q tiles
// (double-buffered over items) and its K/V tiles through a 3-stage TMA ring.
// Warp 1 + g issues group g's MMAs from one thread: for key tile j, S_g = Q_g
// K_j^T (M=128, N=128, K=64) into the group's TMEM S columns, once the group's
// softmax has written P_g of tile j - 1; then O_g += P_g V_{j-1} (M=128, N=64,
// K=128; P_g read from TMEM as packed bf16, V an N-major shared-memory operand,
// O_g accumulated in TMEM). The tensor pipe runs the two threads' instructions
// concurrently (one thread's instructions run one after another, about 120
// cycles each at N <= 128), so each group's S and PV do not queue behind the
// other group's.
// Warps 3..6 (group 0) and 7..10 (group 1) are the softmax warps: thread = query
// row (TMEM lane) with all 128 keys of S_g in registers. The running row max m
// is raised only when a tile's max exceeds it by more than FW_RESCALE (log2
// units); then O (in TMEM) and l are rescaled by 2^(m_old - m_new). Otherwise P
// = 2^(s - m) stays below 2^FW_RESCALE and O / l is the same in exact
// arithmetic. P goes to TMEM as bf16 pairs; the row sum l (fp32, of the
// unrounded exponentials) stays in a register. At an item's end each thread
// reads its O row from TMEM, divides by l and writes it through a
// shared-memory staging tile in 128-byte rows.
// Every wait is bounded (2 s) and reports a timeout in the status word.
#include <cudaTypedefs.h>

#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace gpt2 {

namespace {

constexpr int HD = 64;
constexpr int BQ = 128, BKV = 128;
constexpr int KV_STAGES = 3;
constexpr int FW_THREADS = 96 + 32 * 8;           // TMA warp, two MMA warps, two softmax warpgroups
constexpr int TILE_BYTES = 128 * HD * 2;          // 16 KB: 128 rows x 128 bytes
constexpr float LOG2E = 1.4426950408889634f;
constexpr float FW_RESCALE = 8.f;                 // growth of the row max (log2 units) that triggers a rescale
// TMEM columns of group g, from g * FT_GROUP: S (128 fp32), P (128 keys as bf16
// pairs), O (64 fp32)
constexpr uint32_t FT_S = 0, FT_P = 128, FT_O = 192, FT_GROUP = 256;

struct FwCtl {
    uint64_t q_full[2], q_empty[2];               // Q sets (both groups' tiles of one item); empty: count 2
    uint64_t kv_full[KV_STAGES], kv_empty[KV_STAGES];   // empty: one release per MMA thread
    uint64_t s_full[2];                           // per group: S of its current tile is in TMEM
    uint64_t p_full[2];                           // per group: P written to TMEM (its 4 warps arrive)
    uint64_t pv_done[2];                          // per group: O += P V of its latest tile is done
    uint64_t drain[2];
    uint32_t tmem_base;
    uint32_t abort;
};

// smem: Q[2 sets x 2 groups] | K[3] | V[3] | output staging [2 groups] | ctl
constexpr int FW_OFF_Q = 0;
constexpr int FW_OFF_K = 4 * TILE_BYTES;
constexpr int FW_OFF_V = FW_OFF_K + KV_STAGES * TILE_BYTES;
constexpr int FW_OFF_ST = FW_OFF_V + KV_STAGES * TILE_BYTES;
constexpr int FW_OFF_CTL = FW_OFF_ST + 2 * TILE_BYTES;
constexpr size_t FW_SMEM = FW_OFF_CTL + sizeof(FwCtl) + 1024;

__device__ __forceinline__ uint32_t swz128(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

// 2^x with the hardware approximation (ex2.approx; 2^-inf = 0). Its relative
// error (about 2^-22) is far below the bf16 rounding of P and dS.
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}


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

// Work item i: head-sequence i % BH and query-tile pair n_pairs - 1 - i / BH
// (longest causal prefixes first). Group g's tile starts at q0 + 128 g and uses
// key tiles 0 .. n[g] - 1 (n[1] = 0 when that tile lies past Tn); the item walks
// n_kv = max(n[0], n[1]) key tiles.
struct FwItem {
    int bh, q0, n_kv;
    int n[2];
};
__device__ __forceinline__ FwItem fw_item(int i, int BH, int n_pairs, int Tn) {
    FwItem it;
    it.bh = i % BH;
    it.q0 = (n_pairs - 1 - i / BH) * 2 * BQ;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        const int q = it.q0 + g * BQ;
        it.n[g] = q < Tn ? (min(Tn, q + BQ) + BKV - 1) / BKV : 0;
    }
    it.n_kv = max(it.n[0], it.n[1]);
    return it;
}

// The item this CTA takes in round k (rounds of gridDim.x items, dealt in
// alternating direction so that the longest and shortest even out), or -1.
__device__ __forceinline__ int fw_round_item(int k, int n_items) {
    const int G = gridDim.x;
    const int i = k * G + ((k & 1) ? G - 1 - (int)blockIdx.x : (int)blockIdx.x);
    return i < n_items ? i : -1;
}

// Lane 0 waits on the mbarrier phase; the whole warp gets the result.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile uint32_t* abort,
                                          unsigned* status) {
    uint32_t w = 0;
    if ((threadIdx.x & 31) == 0) w = tc::mbar_wait(bar, parity, abort, status) ? 1u : 0u;
    return __shfl_sync(0xffffffffu, w, 0) != 0;
}

__global__ void __launch_bounds__(FW_THREADS, 1)
    flash_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, bf16* __restrict__ out, float* __restrict__ lse,
                        int Tn, int H, int BH, unsigned* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    FwCtl* ctl = reinterpret_cast<FwCtl*>(smem + FW_OFF_CTL);
    volatile uint32_t* abort = &ctl->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_qt = (Tn + BQ - 1) / BQ;
    const int n_pairs = (n_qt + 1) / 2;
    const int n_items = BH * n_pairs;
    const int n_rounds = (n_items + (int)gridDim.x - 1) / (int)gridDim.x;
    const int C = H * HD;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&ctl->q_full[i], 1);
            tc::mbar_init(&ctl->q_empty[i], 2);
            tc::mbar_init(&ctl->s_full[i], 1);
            tc::mbar_init(&ctl->p_full[i], 4);
            tc::mbar_init(&ctl->pv_done[i], 1);
            tc::mbar_init(&ctl->drain[i], 1);
        }
        for (int s = 0; s < KV_STAGES; ++s) {
            tc::mbar_init(&ctl->kv_full[s], 1);
            tc::mbar_init(&ctl->kv_empty[s], 2);
        }
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
            uint32_t gs = 0;                          // K/V step counter over all items
            uint32_t ord = 0;                         // item counter (Q set ring)
            bool ok = true;
            for (int k = 0; k < n_rounds && ok; ++k) {
                const int i = fw_round_item(k, n_items);
                if (i < 0) continue;
                const FwItem it = fw_item(i, BH, n_pairs, Tn);
                const int row_base = (it.bh / H) * Tn, h = it.bh % H;
                const int qs = ord & 1;
                if (!tc::mbar_wait(&ctl->q_empty[qs], ((ord >> 1) & 1) ^ 1, abort, status)) break;
                tc::mbar_expect_tx(&ctl->q_full[qs], 2 * TILE_BYTES);
                // the second tile may lie past Tn (then unused; rows past the tensor read as zero)
                for (int g = 0; g < 2; ++g)
                    tc::tma_load_2d(smem + FW_OFF_Q + (2 * qs + g) * TILE_BYTES, &tm_qkv, h * HD,
                                    row_base + it.q0 + g * BQ, &ctl->q_full[qs]);
                for (int j = 0; j < it.n_kv; ++j, ++gs) {
                    const int s = gs % KV_STAGES;
                    const uint32_t ph = (gs / KV_STAGES) & 1;
                    if (!tc::mbar_wait(&ctl->kv_empty[s], ph ^ 1, abort, status)) { ok = false; break; }
                    tc::mbar_expect_tx(&ctl->kv_full[s], 2 * TILE_BYTES);
                    tc::tma_load_2d(smem + FW_OFF_K + s * TILE_BYTES, &tm_qkv, C + h * HD, row_base + j * BKV,
                                    &ctl->kv_full[s]);
                    tc::tma_load_2d(smem + FW_OFF_V + s * TILE_BYTES, &tm_qkv, 2 * C + h * HD, row_base + j * BKV,
                                    &ctl->kv_full[s]);
                }
                ++ord;
            }
        }
    } else if (warp <= 2) {
        if (lane == 0) {
            // ------------------------------------------------ MMA, one thread per group
            // Thread g walks every K/V step of the CTA's items in the producer's order.
            // A K/V stage and a Q set are free once both threads have released them, so
            // each thread releases every step and every item, also those its group does
            // not use, and in step order: it waits for a step's fill before releasing it
            // and releases its pending tile (S issued, PV not yet) before any later step.
            const int g = warp - 1;
            constexpr uint32_t idesc_s = tc::idesc_bf16_f32(BQ, BKV, 0, 0);
            constexpr uint32_t idesc_pv = tc::idesc_bf16_f32(BQ, HD, 0, 1);
            const uint32_t tSg = tmem + g * FT_GROUP + FT_S;
            const uint32_t tPg = tmem + g * FT_GROUP + FT_P;
            const uint32_t tOg = tmem + g * FT_GROUP + FT_O;
            uint32_t gs = 0, ord = 0, tp = 0;    // K/V steps, items, PV MMAs issued
            int pend = -1;                       // stage of the pending tile (-1: none)
            bool pend_first = false;             // the pending tile is its item's first: PV overwrites O
            bool ok = true;
            for (int k = 0; k < n_rounds && ok; ++k) {
                const int i = fw_round_item(k, n_items);
                if (i < 0) continue;
                const FwItem it = fw_item(i, BH, n_pairs, Tn);
                const int ng = g == 0 ? it.n[0] : it.n[1];   // this group's key tiles
                const int qs = ord & 1;
                if (!tc::mbar_wait(&ctl->q_full[qs], (ord >> 1) & 1, abort, status)) { ok = false; break; }
                for (int j = 0; j < it.n_kv; ++j, ++gs) {
                    const int s = gs % KV_STAGES;
                    const bool mine = j < ng;
                    if (!tc::mbar_wait(&ctl->kv_full[s], (gs / KV_STAGES) & 1, abort, status)) { ok = false; break; }
                    // the pending tile's P is written (and its S read) before S is overwritten
                    if (pend >= 0 && !tc::mbar_wait(&ctl->p_full[g], tp & 1, abort, status)) { ok = false; break; }
                    tc::fence_after_sync();
                    if (mine) {
                        const uint32_t q_addr = tc::smem_u32(smem + FW_OFF_Q + (2 * qs + g) * TILE_BYTES);
                        const uint32_t k_addr = tc::smem_u32(smem + FW_OFF_K + s * TILE_BYTES);
#pragma unroll
                        for (int kk = 0; kk < HD / 16; ++kk)
                            tc::mma_bf16(tSg, tc::smem_desc_sw128(q_addr + kk * 32, 16, 1024),
                                         tc::smem_desc_sw128(k_addr + kk * 32, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
                        tc::mma_commit(&ctl->s_full[g]);
                        if (j == ng - 1) tc::mma_commit(&ctl->q_empty[qs]);   // the group's last S of the item
                    }
                    if (pend >= 0) {
                        const uint32_t v_addr = tc::smem_u32(smem + FW_OFF_V + pend * TILE_BYTES);
#pragma unroll
                        for (int kk = 0; kk < BKV / 16; ++kk)
                            tc::mma_bf16_ts(tOg, tPg + kk * 8, tc::smem_desc_sw128(v_addr + kk * 2048, TILE_BYTES, 1024),
                                            idesc_pv, (!pend_first || kk > 0) ? 1u : 0u);
                        tc::mma_commit(&ctl->pv_done[g]);
                        tc::mma_commit(&ctl->kv_empty[pend]);
                        ++tp;
                        pend = -1;
                    }
                    if (mine) {
                        pend = s;
                        pend_first = j == 0;
                    } else {
                        tc::mma_commit(&ctl->kv_empty[s]);   // a step this group does not use
                    }
                }
                if (!ok) break;
                if (ng == 0) tc::mma_commit(&ctl->q_empty[qs]);
                ++ord;
            }
            if (ok && pend >= 0 && tc::mbar_wait(&ctl->p_full[g], tp & 1, abort, status)) {
                tc::fence_after_sync();
                const uint32_t v_addr = tc::smem_u32(smem + FW_OFF_V + pend * TILE_BYTES);
#pragma unroll
                for (int kk = 0; kk < BKV / 16; ++kk)
                    tc::mma_bf16_ts(tOg, tPg + kk * 8, tc::smem_desc_sw128(v_addr + kk * 2048, TILE_BYTES, 1024),
                                    idesc_pv, (!pend_first || kk > 0) ? 1u : 0u);
                tc::mma_commit(&ctl->pv_done[g]);
                tc::mma_commit(&ctl->kv_empty[pend]);
            }
            volatile uint32_t no_abort = 0;
            tc::mma_commit(&ctl->drain[g]);
            tc::mbar_wait(&ctl->drain[g], 0, &no_abort, status);
        }
    } else {
        // ---------------------------------------------------- softmax / output
        const int g = (warp - 3) >> 2;
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;            // query row within the tile = TMEM lane
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t tS = tmem + g * FT_GROUP + FT_S + lane_off;
        const uint32_t tP = tmem + g * FT_GROUP + FT_P + lane_off;
        const uint32_t tO = tmem + g * FT_GROUP + FT_O + lane_off;
        const float sl2 = LOG2E * 0.125f;             // log2(e) / sqrt(64)
        uint8_t* stage = smem + FW_OFF_ST + g * TILE_BYTES;
        bool ok = true;
        uint32_t tg = 0;                              // this group's tiles so far
        for (int k = 0; k < n_rounds && ok; ++k) {
            const int i = fw_round_item(k, n_items);
            if (i < 0) continue;
            const FwItem it = fw_item(i, BH, n_pairs, Tn);
            const int n = it.n[g];
            if (n == 0) continue;
            const int q0 = it.q0 + g * BQ;
            const int q = q0 + r;
            float m = 0.f, l = 0.f;
            for (int j = 0; j < n; ++j, ++tg) {
                if (!warp_wait(&ctl->s_full[g], tg & 1, abort, status)) { ok = false; break; }
                tc::fence_after_sync();
                // pass 1: the row max over the tile's 128 keys, 64 columns at a time
                const int kbase = j * BKV;
                const bool diag = kbase + BKV > q0;   // keys after the query do not count
                float mx = -INFINITY;
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    float sv[64];
                    tc::tmem_ld_32x32b_x64(tS + 64 * hh, sv);
                    if (diag) {
#pragma unroll
                        for (int e = 0; e < 64; ++e)
                            if (kbase + 64 * hh + e > q) sv[e] = -INFINITY;
                    }
                    mx = max32(sv + 32, max32(sv, mx));
                }
                const float mt = mx * sl2;
                bool need = false;
                if (j == 0) m = mt;   // the first tile's PV overwrites O
                else need = mt > m + FW_RESCALE;
                // P's TMEM columns and O: the group's previous O += P V must be done
                if (tg > 0) {
                    if (!warp_wait(&ctl->pv_done[g], (tg - 1) & 1, abort, status)) { ok = false; break; }
                    tc::fence_after_sync();
                }
                if (__any_sync(0xffffffffu, need)) {
                    const float cr = need ? ex2(m - mt) : 1.f;
                    if (need) {
                        m = mt;
                        l *= cr;
                    }
#pragma unroll 1
                    for (int hh = 0; hh < 2; ++hh) {
                        float o[32];
                        uint32_t ow[16];
                        tc::tmem_ld_32x32b_x32(tO + 32 * hh, o);
#pragma unroll
                        for (int hq = 0; hq < 2; ++hq) {
#pragma unroll
                            for (int d = 0; d < 16; ++d) ow[d] = __float_as_uint(o[16 * hq + d] * cr);
                            tc::tmem_st_32x32b_x16(tO + 32 * hh + 16 * hq, ow);
                        }
                    }
                }
                // pass 2: P = 2^(s sl2 - m), 64 keys per load: row sum, bf16 pairs into TMEM
                const f32x2 SL = pk2(sl2, sl2), NM = pk2(-m, -m);
                f32x2 RS = pk2(0.f, 0.f);
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    float sv[64];
                    tc::tmem_ld_32x32b_x64(tS + 64 * hh, sv);
                    if (diag) {
#pragma unroll
                        for (int e = 0; e < 64; ++e)
                            if (kbase + 64 * hh + e > q) sv[e] = -INFINITY;
                    }
#pragma unroll
                    for (int cq = 0; cq < 2; ++cq) {
                        float* v = sv + 32 * cq;
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            float t0, t1;
                            upk2(fma2(pk2(v[e], v[e + 1]), SL, NM), t0, t1);
                            v[e] = ex2(t0);
                            v[e + 1] = ex2(t1);
                            RS = add2(RS, pk2(v[e], v[e + 1]));
                        }
                        uint32_t pw[16];
#pragma unroll
                        for (int gq = 0; gq < 4; ++gq) {
                            const uint4 a = pack8_bf16(v + 8 * gq);
                            pw[4 * gq] = a.x; pw[4 * gq + 1] = a.y; pw[4 * gq + 2] = a.z; pw[4 * gq + 3] = a.w;
                        }
                        tc::tmem_st_32x32b_x16(tP + 32 * hh + 16 * cq, pw);
                    }
                }
                tc::tmem_wait_st();
                float rs0, rs1;
                upk2(RS, rs0, rs1);
                l += rs0 + rs1;
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&ctl->p_full[g]);
            }
            if (!ok) break;
            // the item's O is complete once the PV of its last tile is done
            if (!warp_wait(&ctl->pv_done[g], (tg - 1) & 1, abort, status)) { ok = false; break; }
            tc::fence_after_sync();
            {
                float o[64];
                tc::tmem_ld_32x32b_x64(tO, o);
                const float inv = 1.f / l;
#pragma unroll
                for (int gg = 0; gg < 8; ++gg) {
                    float t[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) t[e] = o[8 * gg + e] * inv;
                    *reinterpret_cast<uint4*>(stage + swz128(r, gg)) = pack8_bf16(t);
                }
            }
            if (q < Tn) lse[(long long)it.bh * Tn + q] = (m + log2f(l)) / LOG2E;
            __syncwarp();
            // this warp's 32 rows out, 8 lanes per 128-byte row
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
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

// ============================================================================
// Backward. With P = exp(S - lse) recomputed from the saved lse and
// D = rowsum(dO * O) from the pre-pass:
//   dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),
//   dK = dS^T Q / sqrt(64),  dQ = dS K / sqrt(64).
// One CTA per (b, h, 128-key tile) walks the 128-query tiles at or after its
// key tile, so each (key tile, query tile) pair computes S and dP once:
//   S^T = K Q^T and dP^T = V dO^T (M = 128 keys, N = 128 queries, K = 64) into
//     TMEM (one buffer each; the element-wise warps copy them to registers
//     and release them at once, so the next pair's MMAs run during the
//     element-wise math of this one);
//   8 element-wise warps (thread = key row) form P^T, written to TMEM as the
//     packed-bf16 A operand of dV += P^T dO, and dS^T, written to shared memory
//     (128-byte swizzle, two 64-query atoms): K-major it is the A operand of
//     dK += dS^T Q, MN-major the A operand of dQ = dS K;
//   dV and dK accumulate in TMEM over the query tiles; the pair's dQ (M = 128
//     queries, N = 64) goes to TMEM, and 4 drain warps scale it, stage it in
//     shared memory and add it into an fp32 (B T, C) accumulator with the TMA
//     bulk reduce-add (zeroed by the pre-pass; the post-pass rounds it to
//     bf16 into dqkv).
// Two threads issue the MMAs: warp 1 dV, dQ and dK of each pair, warp 14 the
// S^T and dP^T of the next, so the tensor pipe runs the two streams side by
// side instead of one after the other.
// The 5 matrix products of the algorithm are each computed once; no T x T
// matrix goes to HBM.
// ============================================================================
constexpr int T128_BYTES = 128 * HD * 2;    // 16 KB: 128 rows x 128 bytes

// Rows of a 64-column bf16 result pass through a 128-row staging tile (128
// bytes per row, 128-byte swizzle): each thread writes 32 columns of its own row
// at a time (stage_row_32), then its warp copies whole rows of its 32-row group
// to global memory (flush_rows_64): dst(row) = base + row * ld (elements), rows
// >= n_rows skipped. If csum is non-null, the warp also writes the column sums
// of its 32 rows (rows at or beyond n_rows excluded) of the stored bf16 values
// as 64 floats at csum; a warp whose rows all lie beyond n_rows writes nothing.
__device__ __forceinline__ void stage_row_32(uint8_t* stage, int r, const float* v, float scale, int half) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        float t[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) t[e] = v[8 * c + e] * scale;
        *reinterpret_cast<uint4*>(stage + swz128(r, 4 * half + c)) = pack8_bf16(t);
    }
}
__device__ __forceinline__ void flush_rows_64(const uint8_t* stage, bf16* base, long long ld, int n_rows,
                                              float* csum) {
    const int lane = threadIdx.x & 31, quarter = (threadIdx.x >> 5) & 3;
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

constexpr int BW_EW_WARPS = 8;         // 2 per TMEM lane quarter, 64 query columns each (two chunks of 32)
constexpr int BW_DR_WARPS = 4;         // dQ drain and dK/dV write-out: one per TMEM lane quarter
constexpr int BW_THREADS = 64 + 32 * (BW_EW_WARPS + BW_DR_WARPS) + 32;
constexpr int BW_SDP_WARP = 2 + BW_EW_WARPS + BW_DR_WARPS;   // the thread that issues S^T and dP^T
constexpr int BW_STAGES = 3;           // Q/dO ring
constexpr int BW_ITEM_READERS = 2 + BW_EW_WARPS + BW_DR_WARPS;   // two MMA threads, element-wise and drain warps
struct CtlBwd {
    uint64_t item_full[2], item_empty[2];            // work-item ring, filled by the producer warp
    uint64_t kv_full[2], kv_empty[2];                // K and V of the item in ring slot s
    uint64_t q_full[BW_STAGES], q_empty[BW_STAGES];  // Q, dO, lse and D of one query tile
    uint64_t st_full, st_empty;                      // S^T and dP^T in TMEM: computed / copied to registers
    uint64_t ew_done;                                // P^T (TMEM) and dS^T (shared memory) written
    uint64_t pt_free;                                // a pair's dV MMAs done: P^T reusable
    uint64_t ds_free;                                // a pair's dK, dQ MMAs done: dS^T reusable
    uint64_t dq_full, dq_empty;                      // a pair's dQ in TMEM: computed / copied to registers
    uint64_t acc_done, dkv_free;                     // an item's dK, dV complete in TMEM / copied out
    uint64_t drain[2];                               // per MMA thread
    uint32_t tmem_base;
    uint32_t abort;
    int item[2];
};
// smem: K/V (2 ring slots) | stages x (Q | dO) | dS^T (two 64-query atoms) |
//       staging (per drain warp 32 rows x 128 bytes) | stages x (-lse log2(e) | -D) | ctl
constexpr int BW_KV_BYTES = 2 * T128_BYTES;
constexpr int BW_STAGE_BYTES = 2 * T128_BYTES;
constexpr int BW_DS_BYTES = 2 * T128_BYTES;
constexpr int BW_OFF_KV = 0;
constexpr int BW_OFF_Q = 2 * BW_KV_BYTES;
constexpr int BW_OFF_DS = BW_OFF_Q + BW_STAGES * BW_STAGE_BYTES;
constexpr int BW_OFF_STG = BW_OFF_DS + BW_DS_BYTES;
constexpr int BW_OFF_LSE = BW_OFF_STG + T128_BYTES;  // per stage: 128 floats of -lse log2(e), 128 of -D
constexpr int BW_OFF_CTL = BW_OFF_LSE + BW_STAGES * 1024;
constexpr size_t BW_SMEM = BW_OFF_CTL + sizeof(CtlBwd) + 1024;
// TMEM columns: S^T, dP^T (fp32, 128 queries each), P^T (packed bf16: 128
// queries in 64 columns), the dV and dK accumulators, the pair's dQ.
constexpr uint32_t BW_ST = 0, BW_DPT = 128, BW_PT = 256, BW_DV = 320, BW_DK = 384, BW_DQ = 448;

// Work item i (longest first): key tile i / BH of head-sequence i % BH; its
// query tiles are kt .. n_qt - 1.
struct BwItem {
    int bh, kt, n_it;
};
__device__ __forceinline__ BwItem bw_item(int i, int BH, int n_qt) {
    BwItem w;
    w.kt = i / BH;
    w.bh = i - w.kt * BH;
    w.n_it = n_qt - w.kt;
    return w;
}
// Item of ring slot ictr & 1 (waits for the producer, then frees the slot for
// this reader): the item index, -1 when the work is done, -2 after a failed wait.
__device__ __forceinline__ int bw_read_item(CtlBwd* ctl, uint32_t ictr, volatile uint32_t* abort, unsigned* status) {
    const int s = ictr & 1;
    if (!tc::mbar_wait(&ctl->item_full[s], (ictr >> 1) & 1, abort, status)) return -2;
    const int item = *reinterpret_cast<volatile int*>(&ctl->item[s]);
    tc::mbar_arrive(&ctl->item_empty[s]);
    return item;
}
// The same for a warp: lane 0 reads, every lane gets the value.
__device__ __forceinline__ int bw_read_item_warp(CtlBwd* ctl, uint32_t ictr, volatile uint32_t* abort,
                                                 unsigned* status) {
    int item = 0;
    if ((threadIdx.x & 31) == 0) item = bw_read_item(ctl, ictr, abort, status);
    return __shfl_sync(0xffffffffu, item, 0);
}

// Persistent: gridDim.x CTAs (at most one per SM) take work items in order
// from the counter *work (zeroed by the pre-pass); the producer warp fetches
// the next item's K, V and first query tiles while the current one runs, and
// every ring and barrier parity runs on counters over all of the CTA's pairs.
__global__ void __launch_bounds__(BW_THREADS, 1)
    flash_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_do,
                        const __grid_constant__ CUtensorMap tm_dq, const float* __restrict__ lse,
                        const float* __restrict__ dpre, bf16* __restrict__ dqkv, int Tn, int H, int BH,
                        int* __restrict__ work, float* __restrict__ colsum_part, unsigned* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    CtlBwd* ctl = reinterpret_cast<CtlBwd*>(smem + BW_OFF_CTL);
    volatile uint32_t* abort = &ctl->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = H * HD;
    const int n_qt = (Tn + 127) / 128;
    const int n_items = BH * n_qt;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&ctl->item_full[i], 1);
            tc::mbar_init(&ctl->item_empty[i], BW_ITEM_READERS);
            tc::mbar_init(&ctl->kv_full[i], 1);
            tc::mbar_init(&ctl->kv_empty[i], 2);   // released by both MMA threads
        }
        for (int s = 0; s < BW_STAGES; ++s) {
            tc::mbar_init(&ctl->q_full[s], 2);   // the TMA bytes, and the producer's lse / D stores
            tc::mbar_init(&ctl->q_empty[s], 2);
        }
        tc::mbar_init(&ctl->st_full, 1);
        tc::mbar_init(&ctl->st_empty, BW_EW_WARPS);
        tc::mbar_init(&ctl->ew_done, BW_EW_WARPS);
        tc::mbar_init(&ctl->pt_free, 1);
        tc::mbar_init(&ctl->ds_free, 1);
        tc::mbar_init(&ctl->dq_full, 1);
        tc::mbar_init(&ctl->dq_empty, BW_DR_WARPS);
        tc::mbar_init(&ctl->acc_done, 1);
        tc::mbar_init(&ctl->dkv_free, BW_DR_WARPS);
        tc::mbar_init(&ctl->drain[0], 1);
        tc::mbar_init(&ctl->drain[1], 1);
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
        // -------------------------------------------------------------- producer
        // lane 0 takes items and issues the TMA loads; all 32 lanes stage each
        // query tile's lse (negated, log2 units) and D (negated) next to it.
        if (lane == 0) {
            tc::tma_prefetch_desc(&tm_qkv);
            tc::tma_prefetch_desc(&tm_do);
            tc::tma_prefetch_desc(&tm_dq);
        }
        uint32_t ictr = 0, g = 0;
        for (;;) {
            const int s = ictr & 1;
            const uint32_t ph = (ictr >> 1) & 1;
            int item = -2;
            if (lane == 0 && tc::mbar_wait(&ctl->item_empty[s], ph ^ 1, abort, status)) {
                const int i = atomicAdd(work, 1);
                item = i < n_items ? i : -1;
                ctl->item[s] = item;
                tc::mbar_arrive(&ctl->item_full[s]);
            }
            item = __shfl_sync(0xffffffffu, item, 0);
            if (item < 0) break;
            const BwItem w = bw_item(item, BH, n_qt);
            const int b = w.bh / H, h = w.bh % H, row_base = b * Tn;
            // lse (negated, log2 units) and D (negated) of one query tile, 4 queries per
            // lane, loaded one tile ahead of their stage so that their latency overlaps
            // the wait for the stage
            float nl[4], nd[4];
            auto fetch = [&](int it) {
                const int q0 = (w.kt + it) * 128;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int q = q0 + lane + 32 * j;
                    nl[j] = q < Tn ? lse[(long long)w.bh * Tn + q] : INFINITY;
                    nd[j] = q < Tn ? dpre[(long long)w.bh * Tn + q] : 0.f;
                }
            };
            fetch(0);
            uint32_t ok = 0;
            if (lane == 0 && tc::mbar_wait(&ctl->kv_empty[s], ph ^ 1, abort, status)) {
                uint8_t* kv = smem + BW_OFF_KV + s * BW_KV_BYTES;
                tc::mbar_expect_tx(&ctl->kv_full[s], 2 * T128_BYTES);
                tc::tma_load_2d(kv, &tm_qkv, C + h * HD, row_base + w.kt * 128, &ctl->kv_full[s]);
                tc::tma_load_2d(kv + T128_BYTES, &tm_qkv, 2 * C + h * HD, row_base + w.kt * 128, &ctl->kv_full[s]);
                ok = 1;
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);   // every exit of this loop is taken by the whole warp
            if (!ok) break;
            ++ictr;
            for (int it = 0; it < w.n_it; ++it, ++g) {
                const int st = g % BW_STAGES;
                const int q0 = (w.kt + it) * 128;
                uint8_t* stg = smem + BW_OFF_Q + st * BW_STAGE_BYTES;
                ok = 0;
                if (lane == 0 && tc::mbar_wait(&ctl->q_empty[st], ((g / BW_STAGES) & 1) ^ 1, abort, status)) {
                    tc::mbar_expect_tx(&ctl->q_full[st], 2 * T128_BYTES);
                    tc::tma_load_2d(stg, &tm_qkv, h * HD, row_base + q0, &ctl->q_full[st]);
                    tc::tma_load_2d(stg + T128_BYTES, &tm_do, h * HD, row_base + q0, &ctl->q_full[st]);
                    ok = 1;
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                float* sl = reinterpret_cast<float*>(smem + BW_OFF_LSE + st * 1024);
                float* sd = sl + 128;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    sl[lane + 32 * j] = -nl[j] * LOG2E;   // a query past the sequence: -inf, so P = 0
                    sd[lane + 32 * j] = -nd[j];
                }
                if (it + 1 < w.n_it) fetch(it + 1);
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&ctl->q_full[st]);
            }
            if (!ok) break;
        }
        // before the CTA exits, every load it issued has landed (bounded; at once normally)
        if (lane == 0) {
            volatile uint32_t no_abort = 0;
            for (uint32_t x = ictr > 2 ? ictr - 2 : 0; x < ictr; ++x)
                tc::mbar_wait(&ctl->kv_full[x & 1], (x >> 1) & 1, &no_abort, status);
            for (uint32_t x = g > BW_STAGES ? g - BW_STAGES : 0; x < g; ++x)
                tc::mbar_wait(&ctl->q_full[x % BW_STAGES], (x / BW_STAGES) & 1, &no_abort, status);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------ MMA: dV, dQ, dK of each pair
            constexpr uint32_t idesc_acc = tc::idesc_bf16_f32(128, 64, 0, 1);  // P^T dO, dS^T Q
            constexpr uint32_t idesc_dq = tc::idesc_bf16_f32(128, 64, 1, 1);   // dS K (dS from the dS^T tile)
            // Shared-memory descriptors, built once: the start address sits in the low bits
            // (address >> 4), so stepping inside a tile adds (byte offset >> 4).
            const uint32_t kv0 = tc::smem_u32(smem + BW_OFF_KV), q_base = tc::smem_u32(smem + BW_OFF_Q);
            const uint64_t d_ds_k = tc::smem_desc_sw128(tc::smem_u32(smem + BW_OFF_DS), 16, 1024);
            const uint64_t d_ds_mn = tc::smem_desc_sw128(tc::smem_u32(smem + BW_OFF_DS), T128_BYTES, 1024);
            auto kdesc_mn = [&](int slot) {
                return tc::smem_desc_sw128(kv0 + slot * BW_KV_BYTES, T128_BYTES, 1024);
            };
            auto qdesc_mn = [&](int st) {
                return tc::smem_desc_sw128(q_base + st * BW_STAGE_BYTES, T128_BYTES, 1024);
            };
            constexpr uint64_t TILE16 = T128_BYTES >> 4;   // descriptor step of one 16 KB tile
            uint32_t ictr = 0, g = 0;
            int item = bw_read_item(ctl, ictr, abort, status);
            BwItem cur = bw_item(item < 0 ? 0 : item, BH, n_qt);
            bool ok = item >= 0;
            while (ok) {
                const int slot = ictr & 1;
                // K, V of the item (read by dQ), as filled for this thread's MMAs
                if (!tc::mbar_wait(&ctl->kv_full[slot], (ictr >> 1) & 1, abort, status)) break;
                const uint64_t kmn = kdesc_mn(slot);
                for (int it = 0; it < cur.n_it && ok; ++it, ++g) {
                    const int st = g % BW_STAGES;
                    const uint32_t par = g & 1;
                    // Q and dO of the pair (read by dK and dV), then its P^T and dS^T
                    if (!tc::mbar_wait(&ctl->q_full[st], (g / BW_STAGES) & 1, abort, status) ||
                        !tc::mbar_wait(&ctl->ew_done, par, abort, status)) {
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
                    const uint64_t dmn = qdesc_mn(st);
                    // dQ = dS K: K = 128 keys in steps of 16; A is the dS^T tile read as an MN-major
                    // (query-contiguous) operand, the next 64 queries one atom (16 KB) further
                    auto issue_dq = [&]() -> bool {
                        if (!tc::mbar_wait(&ctl->dq_empty, par ^ 1, abort, status)) return false;
                        tc::fence_after_sync();
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            tc::mma_bf16(tmem + BW_DQ, d_ds_mn + 128 * kk, kmn + 128 * kk, idesc_dq,
                                         kk > 0 ? 1u : 0u);
                        tc::mma_commit(&ctl->dq_full);
                        return true;
                    };
                    // The first pair of an item overwrites dV / dK, so it waits for the last item's
                    // to be copied out; its dQ, which needs neither, goes first. Later pairs issue
                    // dQ right after dV, before dK, so the drain warps can start on it sooner.
                    if (it == 0) {
                        if (!issue_dq() || !tc::mbar_wait(&ctl->dkv_free, (ictr & 1) ^ 1, abort, status)) {
                            ok = false;
                            break;
                        }
                        tc::fence_after_sync();
                    }
                    // dV += P^T dO, then dK += dS^T Q: K = 128 queries in steps of 16
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_bf16_ts(tmem + BW_DV, tmem + BW_PT + kk * 8, dmn + TILE16 + 128 * kk, idesc_acc,
                                        (it > 0 || kk > 0) ? 1u : 0u);
                    tc::mma_commit(&ctl->pt_free);
                    if (it > 0 && !issue_dq()) {
                        ok = false;
                        break;
                    }
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_bf16(tmem + BW_DK, d_ds_k + (kk >> 2) * TILE16 + 2 * (kk & 3), dmn + 128 * kk,
                                     idesc_acc, (it > 0 || kk > 0) ? 1u : 0u);
                    tc::mma_commit(&ctl->q_empty[st]);
                    tc::mma_commit(&ctl->ds_free);
                    if (it + 1 == cur.n_it) {
                        tc::mma_commit(&ctl->kv_empty[slot]);
                        tc::mma_commit(&ctl->acc_done);
                    }
                }
                if (!ok) break;
                item = bw_read_item(ctl, ++ictr, abort, status);
                if (item < 0) break;
                cur = bw_item(item, BH, n_qt);
            }
            volatile uint32_t no_abort = 0;
            tc::mma_commit(&ctl->drain[0]);
            tc::mbar_wait(&ctl->drain[0], 0, &no_abort, status);
        }
    } else if (warp < 2 + BW_EW_WARPS) {
        // --------------------------------------------- P^T, dS^T (thread = key row)
        const int quarter = warp & 3;
        const int chalf = (warp - 2) >> 2;              // query columns [64 chalf, 64 chalf + 64)
        const int r = quarter * 32 + lane;              // key row in the tile = TMEM lane
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const float sl2 = LOG2E * 0.125f;
        const int qa = chalf * 64;
        // P^T = 2^(s sl2 - lse2), dS^T = P^T (dP^T - D) for the 32 queries from qc, in
        // place (sv becomes P^T, dp becomes dS^T), packed to bf16 pairs
        auto ew_chunk = [&](float* sv, float* dp, const float* sl, const float* sd, int qc, bool diag, uint32_t* pw,
                            uint32_t* dw) {
            const f32x2 SL = pk2(sl2, sl2);
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
                const float4 nl = *reinterpret_cast<const float4*>(sl + qc + e);
                const float4 nd = *reinterpret_cast<const float4*>(sd + qc + e);
                float t0, t1, t2, t3;
                upk2(fma2(pk2(sv[e], sv[e + 1]), SL, pk2(nl.x, nl.y)), t0, t1);
                upk2(fma2(pk2(sv[e + 2], sv[e + 3]), SL, pk2(nl.z, nl.w)), t2, t3);
                sv[e] = ex2(t0);
                sv[e + 1] = ex2(t1);
                sv[e + 2] = ex2(t2);
                sv[e + 3] = ex2(t3);
                if (diag) {   // queries before this key (the diagonal pair: q0 = k0)
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        if (r > qc + e + j) sv[e + j] = 0.f;
                }
                upk2(mul2(pk2(sv[e], sv[e + 1]), add2(pk2(dp[e], dp[e + 1]), pk2(nd.x, nd.y))), dp[e], dp[e + 1]);
                upk2(mul2(pk2(sv[e + 2], sv[e + 3]), add2(pk2(dp[e + 2], dp[e + 3]), pk2(nd.z, nd.w))), dp[e + 2],
                     dp[e + 3]);
            }
#pragma unroll
            for (int gq = 0; gq < 4; ++gq) {
                const uint4 a = pack8_bf16(sv + 8 * gq), d = pack8_bf16(dp + 8 * gq);
                pw[4 * gq] = a.x; pw[4 * gq + 1] = a.y; pw[4 * gq + 2] = a.z; pw[4 * gq + 3] = a.w;
                dw[4 * gq] = d.x; dw[4 * gq + 1] = d.y; dw[4 * gq + 2] = d.z; dw[4 * gq + 3] = d.w;
            }
        };
        uint32_t ictr = 0, g = 0;
        int item = bw_read_item_warp(ctl, ictr, abort, status);
        BwItem cur = bw_item(item < 0 ? 0 : item, BH, n_qt);
        int it = 0;
        while (item >= 0) {
            const int st = g % BW_STAGES;
            const uint32_t par = g & 1;
            uint32_t w = 0;
            if (lane == 0) w = tc::mbar_wait(&ctl->st_full, par, abort, status) ? 1u : 0u;
            if (!__shfl_sync(0xffffffffu, w, 0)) break;
            // the producer's lse / D stores of this stage (complete long before S^T is);
            // every lane acquires them, and the warp leaves together if one lane's wait fails
            w = tc::mbar_wait(&ctl->q_full[st], (g / BW_STAGES) & 1, abort, status) ? 1u : 0u;
            if (!__all_sync(0xffffffffu, w)) break;
            tc::fence_after_sync();
            const float* sl = reinterpret_cast<const float*>(smem + BW_OFF_LSE + st * 1024);
            const float* sd = sl + 128;
            const bool diag = (it == 0);
            uint8_t* ds_tile = smem + BW_OFF_DS + chalf * T128_BYTES;
            bool fail = false;
            uint32_t dw0[16];   // dS^T of chunk 0, kept until the previous pair's dK / dQ MMAs are done
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
                float sv[32], dp[32];
                uint32_t pw[16], dw[16];
                tc::tmem_ld2_32x32b_x32(tmem + BW_ST + qa + 32 * c + lane_off, tmem + BW_DPT + qa + 32 * c + lane_off,
                                        sv, dp);
                if (c == 1) {   // S^T and dP^T are in registers: the next pair's MMAs may overwrite them
                    tc::fence_before_sync();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(&ctl->st_empty);
                }
                ew_chunk(sv, dp, sl, sd, qa + 32 * c, diag, pw, dw);
                // P^T's TMEM columns: the previous pair's dV MMAs are done (chunk 0 waits)
                if (c == 0) {
                    if (lane == 0) w = tc::mbar_wait(&ctl->pt_free, par ^ 1, abort, status) ? 1u : 0u;
                    if (!__shfl_sync(0xffffffffu, w, 0)) { fail = true; break; }
                    tc::fence_after_sync();
                }
                tc::tmem_st_32x32b_x16(tmem + BW_PT + chalf * 32 + 16 * c + lane_off, pw);
                if (c == 0) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) dw0[j] = dw[j];
                } else {
                    // dS^T: the previous pair's dK / dQ MMAs are done
                    if (lane == 0) w = tc::mbar_wait(&ctl->ds_free, par ^ 1, abort, status) ? 1u : 0u;
                    if (!__shfl_sync(0xffffffffu, w, 0)) { fail = true; break; }
                    tc::fence_after_sync();
#pragma unroll
                    for (int gq = 0; gq < 4; ++gq) {
                        *reinterpret_cast<uint4*>(ds_tile + swz128(r, gq)) =
                            make_uint4(dw0[4 * gq], dw0[4 * gq + 1], dw0[4 * gq + 2], dw0[4 * gq + 3]);
                        *reinterpret_cast<uint4*>(ds_tile + swz128(r, 4 + gq)) =
                            make_uint4(dw[4 * gq], dw[4 * gq + 1], dw[4 * gq + 2], dw[4 * gq + 3]);
                    }
                }
            }
            if (fail) break;
            tc::tmem_wait_st();
            tc::fence_proxy_async_smem();      // dS^T visible to the tensor core
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&ctl->ew_done);
            ++g;
            if (++it == cur.n_it) {
                item = bw_read_item_warp(ctl, ++ictr, abort, status);
                if (item >= 0) cur = bw_item(item, BH, n_qt);
                it = 0;
            }
        }
    } else if (warp < BW_SDP_WARP) {
        // ------------------------------- dQ drain, dK / dV write-out (thread = row)
        // Each warp moves its own 32 rows through its own 4 KB of staging: dQ as two
        // fp32 32 x 32 boxes added into the accumulator by this warp's TMA reduce,
        // then at an item's end dK and dV as bf16 rows. No barrier spans warps.
        const int quarter = warp & 3;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int r = quarter * 32 + lane;
        uint8_t* stage = smem + BW_OFF_STG;                   // 128 rows x 128 bytes
        uint8_t* mine = stage + quarter * 4096;               // this warp's rows
        uint32_t ictr = 0, g = 0;
        int item = bw_read_item_warp(ctl, ictr, abort, status);
        BwItem cur = bw_item(item < 0 ? 0 : item, BH, n_qt);
        int it = 0;
        while (item >= 0) {
            const int b = cur.bh / H, h = cur.bh % H, row_base = b * Tn, k0 = cur.kt * 128;
            const int q0 = (cur.kt + it) * 128;
            uint32_t w = 0;
            if (lane == 0) w = tc::mbar_wait(&ctl->dq_full, g & 1, abort, status) ? 1u : 0u;
            if (!__shfl_sync(0xffffffffu, w, 0)) break;
            tc::fence_after_sync();
            const bool live = q0 + quarter * 32 < Tn;          // rows past the sequence add nothing
            // dQ in two 32-column halves: each a fp32 box of 32 rows x 32 columns (128-byte
            // swizzle) added into the accumulator; dQ = dS K / sqrt(64). The TMEM columns
            // are free once the second half is in registers.
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                float v[32];
                tc::tmem_ld_32x32b_x32(tmem + BW_DQ + 32 * half + lane_off, v);
                if (half == 1) {
                    tc::fence_before_sync();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(&ctl->dq_empty);
                }
                if (lane == 0) tc::bulk_wait_read<0>();       // this warp's last reduce has read the staging
                __syncwarp();
#pragma unroll
                for (int cc = 0; cc < 8; ++cc)
                    *reinterpret_cast<float4*>(mine + swz128(lane, cc)) =
                        make_float4(v[4 * cc] * 0.125f, v[4 * cc + 1] * 0.125f, v[4 * cc + 2] * 0.125f,
                                    v[4 * cc + 3] * 0.125f);
                tc::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0 && live) {
                    tc::tma_reduce_add_2d(&tm_dq, mine, h * HD + 32 * half, row_base + q0 + quarter * 32);
                    tc::bulk_commit();
                }
            }
            ++g;
            if (++it == cur.n_it) {
                // the item's dK, dV: TMEM -> bf16 rows (+ column sums), then TMEM is free
                if (lane == 0) w = tc::mbar_wait(&ctl->acc_done, ictr & 1, abort, status) ? 1u : 0u;
                if (!__shfl_sync(0xffffffffu, w, 0)) break;
                tc::fence_after_sync();
                if (lane == 0) tc::bulk_wait_read<0>();
                __syncwarp();
                bf16* kbase = dqkv + ((long long)row_base + k0) * 3 * C + C + h * HD;
                // column sums (the c_attn bias gradient) of this warp's 32-row group
                float* cs = colsum_part
                                ? colsum_part + ((long long)b * ((Tn + 31) / 32) + cur.kt * 4 + quarter) * 3 * C
                                : nullptr;
#pragma unroll 1
                for (int m = 0; m < 2; ++m) {   // dK (scaled by 1 / sqrt(64)), then dV
#pragma unroll 1
                    for (int half = 0; half < 2; ++half) {
                        float v[32];
                        tc::tmem_ld_32x32b_x32(tmem + (m ? BW_DV : BW_DK) + 32 * half + lane_off, v);
                        stage_row_32(stage, r, v, m ? 1.0f : 0.125f, half);
                    }
                    flush_rows_64(stage, kbase + m * C, 3LL * C, Tn - k0, cs ? cs + (m + 1) * C + h * HD : nullptr);
                }
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&ctl->dkv_free);
                item = bw_read_item_warp(ctl, ++ictr, abort, status);
                if (item >= 0) cur = bw_item(item, BH, n_qt);
                it = 0;
            }
        }
        if (lane == 0) tc::bulk_wait<0>();
    } else if (lane == 0) {
        // ----------------------------------------------- MMA: S^T and dP^T of each pair
        // S^T = K Q^T and dP^T = V dO^T (M = 128 keys, N = 128 queries, K = 64) of pair g,
        // once the element-wise warps hold pair g - 1's in registers. This thread and the
        // dV / dQ / dK thread each release the Q/dO stage and the K/V slot they read, and
        // each waits for the fills itself, so every release lands in its own phase.
        constexpr uint32_t idesc_s = tc::idesc_bf16_f32(128, 128, 0, 0);
        constexpr uint64_t TILE16 = T128_BYTES >> 4;
        const uint32_t kv0 = tc::smem_u32(smem + BW_OFF_KV), q_base = tc::smem_u32(smem + BW_OFF_Q);
        uint32_t ictr = 0, g = 0;
        int item = bw_read_item(ctl, ictr, abort, status);
        BwItem cur = bw_item(item < 0 ? 0 : item, BH, n_qt);
        bool ok = item >= 0;
        while (ok) {
            const int slot = ictr & 1;
            if (!tc::mbar_wait(&ctl->kv_full[slot], (ictr >> 1) & 1, abort, status)) break;
            const uint64_t dk = tc::smem_desc_sw128(kv0 + slot * BW_KV_BYTES, 16, 1024);
            for (int it = 0; it < cur.n_it; ++it, ++g) {
                const int st = g % BW_STAGES;
                if ((g > 0 && !tc::mbar_wait(&ctl->st_empty, (g - 1) & 1, abort, status)) ||
                    !tc::mbar_wait(&ctl->q_full[st], (g / BW_STAGES) & 1, abort, status)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                const uint64_t dq = tc::smem_desc_sw128(q_base + st * BW_STAGE_BYTES, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    tc::mma_bf16(tmem + BW_ST, dk + 2 * kk, dq + 2 * kk, idesc_s, kk > 0 ? 1u : 0u);
                    tc::mma_bf16(tmem + BW_DPT, dk + TILE16 + 2 * kk, dq + TILE16 + 2 * kk, idesc_s,
                                 kk > 0 ? 1u : 0u);
                }
                tc::mma_commit(&ctl->st_full);
                tc::mma_commit(&ctl->q_empty[st]);
            }
            if (!ok) break;
            tc::mma_commit(&ctl->kv_empty[slot]);
            item = bw_read_item(ctl, ++ictr, abort, status);
            if (item < 0) break;
            cur = bw_item(item, BH, n_qt);
        }
        volatile uint32_t no_abort = 0;
        tc::mma_commit(&ctl->drain[1]);
        tc::mbar_wait(&ctl->drain[1], 0, &no_abort, status);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

// D = rowsum(dO * O) for every head of one (b, t) row, the fp32 dQ accumulator
// row set to zero, and the work-item counter reset: one warp per row; 8 lanes
// per head (16 bytes of O and of dO each), 4 heads per pass.
__global__ void __launch_bounds__(256) flash_bwd_pre_tc_kernel(const bf16* __restrict__ out,
                                                               const bf16* __restrict__ dout,
                                                               float* __restrict__ dpre, float* __restrict__ dq_acc,
                                                               int* __restrict__ work, int Tn, int H, long long rows) {
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (blockIdx.x == 0 && threadIdx.x == 0) *work = 0;
    if (row >= rows) return;
    const int b = (int)(row / Tn), t = (int)(row % Tn);
    const long long C = (long long)H * HD;
    for (int h0 = 0; h0 < H; h0 += 4) {
        const int h = h0 + (lane >> 3);
        float s = 0.f;
        if (h < H) {
            const long long o = row * C + h * HD + (lane & 7) * 8;
            const uint4 x = *reinterpret_cast<const uint4*>(out + o);
            const uint4 y = *reinterpret_cast<const uint4*>(dout + o);
            const __nv_bfloat162* xa = reinterpret_cast<const __nv_bfloat162*>(&x);
            const __nv_bfloat162* ya = reinterpret_cast<const __nv_bfloat162*>(&y);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 fx = __bfloat1622float2(xa[j]), fy = __bfloat1622float2(ya[j]);
                s = fmaf(fx.x, fy.x, fmaf(fx.y, fy.y, s));
            }
        }
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        s += __shfl_xor_sync(0xffffffffu, s, 4);
        if (h < H && (lane & 7) == 0) dpre[((long long)b * H + h) * Tn + t] = s;
    }
    float4* z = reinterpret_cast<float4*>(dq_acc + row * C);
    for (long long i = lane; i < C / 4; i += 32) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// dq columns of dqkv = the fp32 accumulator rounded to bf16, and (if
// colsum_part) the column sums of each 32-row group of the stored values, in
// row order. Block = one 32-row group of one sequence; thread = 8 columns of
// each blockDim.x * 8 column stretch.
__global__ void __launch_bounds__(256) flash_bwd_dq_post_kernel(const float* __restrict__ dq_acc,
                                                                bf16* __restrict__ dqkv, int Tn, int C,
                                                                float* __restrict__ colsum_part) {
    const int G = (Tn + 31) / 32;
    const int b = blockIdx.x / G, grp = blockIdx.x % G;
    const int t0 = grp * 32, t1 = min(Tn, t0 + 32);
    for (int c0 = threadIdx.x * 8; c0 < C; c0 += blockDim.x * 8) {
    float sum[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) sum[e] = 0.f;
#pragma unroll 4
    for (int t = t0; t < t1; ++t) {
        const long long row = (long long)b * Tn + t;
        const float4 x0 = *reinterpret_cast<const float4*>(dq_acc + row * C + c0);
        const float4 x1 = *reinterpret_cast<const float4*>(dq_acc + row * C + c0 + 4);
        const float v[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
        const uint4 q = pack8_bf16(v);
        *reinterpret_cast<uint4*>(dqkv + row * 3 * C + c0) = q;
        const __nv_bfloat162* qa = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(qa[j]);
            sum[2 * j] += f.x;
            sum[2 * j + 1] += f.y;
        }
    }
    if (colsum_part) {
        float* dst = colsum_part + (long long)blockIdx.x * 3 * C + c0;
        *reinterpret_cast<float4*>(dst) = make_float4(sum[0], sum[1], sum[2], sum[3]);
        *reinterpret_cast<float4*>(dst + 4) = make_float4(sum[4], sum[5], sum[6], sum[7]);
    }
    }
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
        cudaFuncSetAttribute(flash_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)FW_SMEM);
        configured = true;
    }
    const int n_items = B * H * ((ceil_div(Tn, BQ) + 1) / 2);   // query-tile pairs
    const int grid = min(n_items, ctx.num_sms > 0 ? ctx.num_sms : 148);
    flash_fwd_tc_kernel<<<grid, FW_THREADS, FW_SMEM, ctx.stream>>>(m, out, lse, Tn, H, B * H, ctx.status);
    ++*ctx.launches;
    return true;
}

bool launch_attention_bwd_tc(const Ctx& ctx, const bf16* qkv, const bf16* out, const bf16* dout, const float* lse,
                             float* dpre, float* dq_acc, int* work, bf16* dqkv, int B, int Tn, int H,
                             float* colsum_part) {
    auto fn = encode_fn_attn();
    if (!fn) return false;
    const long long C = (long long)H * HD;
    auto make = [&](CUtensorMap* m, CUtensorMapDataType dt, const void* base, long long cols, int esize,
                    int box_cols, int box_rows) {
        cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)B * Tn};
        cuuint64_t strides[1] = {(cuuint64_t)cols * esize};
        cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
        cuuint32_t estr[2] = {1, 1};
        return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    };
    CUtensorMap m_qkv, m_do, m_dq;
    if (!make(&m_qkv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, qkv, 3 * C, 2, 64, 128) ||
        !make(&m_do, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dout, C, 2, 64, 128) ||
        !make(&m_dq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, dq_acc, C, 4, 32, 32))
        return false;
    static bool configured = false;
    if (!configured) {
        cudaFuncSetAttribute(flash_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)BW_SMEM);
        configured = true;
    }
    const long long rows = (long long)B * Tn;
    flash_bwd_pre_tc_kernel<<<(unsigned)ceil_div_ll(rows, 8), 256, 0, ctx.stream>>>(out, dout, dpre, dq_acc, work, Tn,
                                                                                   H, rows);
    const int n_items = B * H * ceil_div(Tn, 128);
    const int grid = min(n_items, ctx.num_sms > 0 ? ctx.num_sms : 148);
    flash_bwd_tc_kernel<<<grid, BW_THREADS, BW_SMEM, ctx.stream>>>(m_qkv, m_do, m_dq, lse, dpre, dqkv, Tn, H, B * H,
                                                                   work, colsum_part, ctx.status);
    flash_bwd_dq_post_kernel<<<B * ceil_div(Tn, 32), (unsigned)min(C / 8, 256LL), 0, ctx.stream>>>(
        dq_acc, dqkv, Tn, (int)C, colsum_part);
    *ctx.launches += 3;
    return true;
}

}  // namespace gpt2
