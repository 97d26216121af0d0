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
// One CTA = one (b, h) and 128 queries (one query per softmax thread and TMEM
// lane). Warp 0 loads Q once and the K/V tiles of the causal prefix through a
// 2-stage TMA ring; warp 1 issues, from one thread, S_j = Q K_j^T (M=128,
// N=128, K=64) into one of two TMEM S buffers and PV_j = P_j V_j (M=128, N=64,
// K=128; V described as an N-major operand) into one of two TMEM PV buffers;
// warps 2..5 read S_j from TMEM (two passes: row max, then exp2 / row sum /
// bf16 P into a 128-byte-swizzled K-major shared tile), then fold PV_{j-1}
// into the register-resident output row: O = O * exp2(m_{j-2} - m_{j-1}) + PV.
// Every wait is bounded (2 s) and reports a timeout in the status word.
#include <cudaTypedefs.h>

#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace gpt2 {

namespace {

constexpr int HD = 64;
constexpr int BQ = 128, BKV = 128;
constexpr int KV_STAGES = 2;
constexpr int THREADS = 192;
constexpr int TILE_BYTES = 128 * HD * 2;          // 16 KB: 128 rows x 128 bytes
constexpr int P_BYTES = BQ * BKV * 2;             // 32 KB: two 64-key swizzle atoms of 16 KB
constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_PV0 = 256, TM_PV1 = 320;
constexpr float LOG2E = 1.4426950408889634f;

struct Ctl {
    uint64_t q_full;
    uint64_t kv_full[KV_STAGES], kv_empty[KV_STAGES];
    uint64_t s_full[2], s_empty[2];
    uint64_t p_full[2];
    uint64_t pv_full[2], pv_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    uint32_t abort;
};

// smem: Q | K[2] | V[2] | P[2] | ctl
constexpr int OFF_Q = 0;
constexpr int OFF_K = OFF_Q + TILE_BYTES;
constexpr int OFF_V = OFF_K + KV_STAGES * TILE_BYTES;
constexpr int OFF_P = OFF_V + KV_STAGES * TILE_BYTES;
constexpr int OFF_CTL = OFF_P + 2 * P_BYTES;
constexpr size_t SMEM_BYTES = OFF_CTL + sizeof(Ctl) + 1024;

__device__ __forceinline__ uint32_t swz128(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

__global__ void __launch_bounds__(THREADS, 1)
    flash_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, bf16* __restrict__ out, float* __restrict__ lse,
                        int Tn, int H, unsigned* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctl* ctl = reinterpret_cast<Ctl*>(smem + OFF_CTL);
    volatile uint32_t* abort = &ctl->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_qt = gridDim.x;
    const int qt = n_qt - 1 - blockIdx.x;            // longest causal prefixes first
    const int bh = blockIdx.y, b = bh / H, h = bh % H;
    const int C = H * HD;
    const int q0 = qt * BQ;
    const int n_kv = (min(Tn, q0 + BQ) + BKV - 1) / BKV;   // key tiles 0 .. n_kv-1
    const int row_base = b * Tn;                      // first row of this sequence in qkv

    if (threadIdx.x == 0) {
        tc::mbar_init(&ctl->q_full, 1);
        for (int s = 0; s < KV_STAGES; ++s) {
            tc::mbar_init(&ctl->kv_full[s], 1);
            tc::mbar_init(&ctl->kv_empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&ctl->s_full[i], 1);
            tc::mbar_init(&ctl->s_empty[i], 4);
            tc::mbar_init(&ctl->p_full[i], 4);
            tc::mbar_init(&ctl->pv_full[i], 1);
            tc::mbar_init(&ctl->pv_empty[i], 4);
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
            tc::mbar_expect_tx(&ctl->q_full, TILE_BYTES);
            tc::tma_load_2d(smem + OFF_Q, &tm_qkv, h * HD, row_base + q0, &ctl->q_full);
            for (int j = 0; j < n_kv; ++j) {
                const int s = j % KV_STAGES;
                const uint32_t ph = (j / KV_STAGES) & 1;
                if (!tc::mbar_wait(&ctl->kv_empty[s], ph ^ 1, abort, status)) break;
                tc::mbar_expect_tx(&ctl->kv_full[s], 2 * TILE_BYTES);
                tc::tma_load_2d(smem + OFF_K + s * TILE_BYTES, &tm_qkv, C + h * HD, row_base + j * BKV,
                                &ctl->kv_full[s]);
                tc::tma_load_2d(smem + OFF_V + s * TILE_BYTES, &tm_qkv, 2 * C + h * HD, row_base + j * BKV,
                                &ctl->kv_full[s]);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // --------------------------------------------------------------- MMA
            constexpr uint32_t idesc_s = tc::idesc_bf16_f32(BQ, BKV, 0, 0);
            constexpr uint32_t idesc_pv = tc::idesc_bf16_f32(BQ, HD, 0, 1);
            const uint32_t q_addr = tc::smem_u32(smem + OFF_Q);
            bool ok = tc::mbar_wait(&ctl->q_full, 0, abort, status);
            auto issue_s = [&](int j) -> bool {
                const int s = j % KV_STAGES, sb = j & 1;
                if (!tc::mbar_wait(&ctl->kv_full[s], (j / KV_STAGES) & 1, abort, status)) return false;
                if (!tc::mbar_wait(&ctl->s_empty[sb], ((j >> 1) & 1) ^ 1, abort, status)) return false;
                tc::fence_after_sync();
                const uint32_t k_addr = tc::smem_u32(smem + OFF_K + s * TILE_BYTES);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk)
                    tc::mma_bf16(tmem + (sb ? TM_S1 : TM_S0), tc::smem_desc_sw128(q_addr + kk * 32, 16, 1024),
                                 tc::smem_desc_sw128(k_addr + kk * 32, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
                tc::mma_commit(&ctl->s_full[sb]);
                return true;
            };
            if (ok && n_kv > 0) ok = issue_s(0);
            for (int j = 0; j < n_kv && ok; ++j) {
                if (j + 1 < n_kv && !issue_s(j + 1)) break;
                const int s = j % KV_STAGES, pb = j & 1;
                if (!tc::mbar_wait(&ctl->p_full[pb], (j >> 1) & 1, abort, status)) break;
                if (!tc::mbar_wait(&ctl->pv_empty[pb], ((j >> 1) & 1) ^ 1, abort, status)) break;
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
            }
            volatile uint32_t no_abort = 0;
            tc::mma_commit(&ctl->drain);
            tc::mbar_wait(&ctl->drain, 0, &no_abort, status);
        }
    } else {
        // ---------------------------------------------------- softmax / output
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;            // query row within the tile = TMEM lane
        const int q = q0 + r;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const float sl2 = LOG2E * 0.125f;             // log2(e) / sqrt(64)
        float o[HD];
#pragma unroll
        for (int d = 0; d < HD; ++d) o[d] = 0.f;
        float m = -INFINITY, l = 0.f, corr_prev = 1.f;
        bool ok = true;
        auto consume_pv = [&](int j) -> bool {
            const int pb = j & 1;
            uint32_t w = 0;
            if (lane == 0) w = tc::mbar_wait(&ctl->pv_full[pb], (j >> 1) & 1, abort, status) ? 1u : 0u;
            w = __shfl_sync(0xffffffffu, w, 0);
            if (!w) return false;
            tc::fence_after_sync();
            float pv[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                tc::tmem_ld_32x32b_x32(tmem + (pb ? TM_PV1 : TM_PV0) + half * 32 + lane_off, pv);
#pragma unroll
                for (int d = 0; d < 32; ++d) o[half * 32 + d] = fmaf(o[half * 32 + d], corr_prev, pv[d]);
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&ctl->pv_empty[pb]);
            return true;
        };
        for (int j = 0; j < n_kv; ++j) {
            const int sb = j & 1;
            uint32_t w = 0;
            if (lane == 0) w = tc::mbar_wait(&ctl->s_full[sb], (j >> 1) & 1, abort, status) ? 1u : 0u;
            w = __shfl_sync(0xffffffffu, w, 0);
            if (!w) { ok = false; break; }
            tc::fence_after_sync();
            const uint32_t s_addr = tmem + (sb ? TM_S1 : TM_S0) + lane_off;
            const bool diag = (j * BKV + BKV > q0);   // tile reaches past the first query of the block
            // pass 1: row max
            float mx = -INFINITY;
#pragma unroll 1
            for (int c = 0; c < BKV; c += 32) {
                float sv[32];
                tc::tmem_ld_32x32b_x32(s_addr + c, sv);
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int key = j * BKV + c + e;
                    if (!diag || key <= q) mx = fmaxf(mx, sv[e]);
                }
            }
            const float m_new = fmaxf(m, mx * sl2);
            const float corr = exp2f(m - m_new);   // m = -inf at the start: 0
            // pass 2: P = exp2(s * sl2 - m_new) as bf16 into the K-major swizzled tile
            uint8_t* pt = smem + OFF_P + sb * P_BYTES;
            float rs = 0.f;
#pragma unroll 1
            for (int c = 0; c < BKV; c += 32) {
                float sv[32];
                tc::tmem_ld_32x32b_x32(s_addr + c, sv);
                float p[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int key = j * BKV + c + e;
                    p[e] = (!diag || key <= q) ? exp2f(fmaf(sv[e], sl2, -m_new)) : 0.f;
                    rs += p[e];
                }
                const int atom = c >> 6;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const int chunk = ((c & 63) >> 3) + g;   // 16-byte chunk within the 128-byte atom row
                    uint4 v;
                    __nv_bfloat162 t0 = __floats2bfloat162_rn(p[8 * g + 0], p[8 * g + 1]);
                    __nv_bfloat162 t1 = __floats2bfloat162_rn(p[8 * g + 2], p[8 * g + 3]);
                    __nv_bfloat162 t2 = __floats2bfloat162_rn(p[8 * g + 4], p[8 * g + 5]);
                    __nv_bfloat162 t3 = __floats2bfloat162_rn(p[8 * g + 6], p[8 * g + 7]);
                    v.x = *reinterpret_cast<uint32_t*>(&t0);
                    v.y = *reinterpret_cast<uint32_t*>(&t1);
                    v.z = *reinterpret_cast<uint32_t*>(&t2);
                    v.w = *reinterpret_cast<uint32_t*>(&t3);
                    *reinterpret_cast<uint4*>(pt + atom * TILE_BYTES + swz128(r, chunk)) = v;
                }
            }
            l = l * corr + rs;
            m = m_new;
            tc::fence_proxy_async_smem();      // P visible to the tensor core
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                tc::mbar_arrive(&ctl->p_full[sb]);
                tc::mbar_arrive(&ctl->s_empty[sb]);
            }
            if (j > 0 && !consume_pv(j - 1)) { ok = false; break; }
            corr_prev = corr;
        }
        if (ok && n_kv > 0) ok = consume_pv(n_kv - 1);
        if (ok) {
            // out row q: O / l, staged through the Q tile (free now) for 128-byte row stores
            const float inv = 1.f / l;
            uint8_t* stage = smem + OFF_Q;
            __syncwarp();
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint4 v;
                __nv_bfloat162 t0 = __floats2bfloat162_rn(o[8 * c + 0] * inv, o[8 * c + 1] * inv);
                __nv_bfloat162 t1 = __floats2bfloat162_rn(o[8 * c + 2] * inv, o[8 * c + 3] * inv);
                __nv_bfloat162 t2 = __floats2bfloat162_rn(o[8 * c + 4] * inv, o[8 * c + 5] * inv);
                __nv_bfloat162 t3 = __floats2bfloat162_rn(o[8 * c + 6] * inv, o[8 * c + 7] * inv);
                v.x = *reinterpret_cast<uint32_t*>(&t0);
                v.y = *reinterpret_cast<uint32_t*>(&t1);
                v.z = *reinterpret_cast<uint32_t*>(&t2);
                v.w = *reinterpret_cast<uint32_t*>(&t3);
                *reinterpret_cast<uint4*>(stage + swz128(r, c)) = v;
            }
            if (q < Tn) lse[(long long)bh * Tn + q] = (m + log2f(l)) / LOG2E;
            __syncwarp();
            const int lrow = lane >> 3, lseg = lane & 7;
#pragma unroll
            for (int st = 0; st < 8; ++st) {
                const int rr = quarter * 32 + st * 4 + lrow;
                if (q0 + rr < Tn)
                    *reinterpret_cast<uint4*>(out + ((long long)b * Tn + q0 + rr) * C + h * HD + lseg * 8) =
                        *reinterpret_cast<const uint4*>(stage + swz128(rr, lseg));
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
    dim3 grid(ceil_div(Tn, BQ), B * H);
    flash_fwd_tc_kernel<<<grid, THREADS, SMEM_BYTES, ctx.stream>>>(m, out, lse, Tn, H, ctx.status);
    ++*ctx.launches;
    return true;
}

}  // namespace gpt2
