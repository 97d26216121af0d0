// Persistent tensor-core GEMM for sm_100a.
//
// One CTA per SM walks a static list of work units (output tile x K split).
// Warp 0 streams A/B k-blocks with TMA into a 4-stage shared-memory ring that
// runs continuously across units; warp 1 issues tcgen05.mma (kind::f16, bf16
// operands, M=128, N=256, K=16) from one thread into one of two fp32
// accumulators in tensor memory (2 x 256 columns = all 512); the epilogue
// warps (from warp 2 on) read the other accumulator with tcgen05.ld and run the
// fused epilogue while the next unit's MMAs proceed, then hand the accumulator
// back. Eight epilogue warps (two per TMEM lane quarter, 128 of the 256 columns
// each) serve the light epilogues; the GELU epilogue, whose arithmetic per
// element is the longest, gets sixteen (four per lane quarter, 64 columns
// each), so each scheduler has four of them to hide its latencies. Each
// epilogue warp turns its rows around in a private swizzled shared-memory
// buffer so that results and epilogue inputs move through global memory as
// 128-byte rows (64-byte row segments for the sixteen-warp layout).
//
// All three operand layouts of the training step run on the same kernel:
//   NT (forward, y = x W^T):   A K-major,  B K-major
//   NN (dgrad,   dx = dy W):   A K-major,  B N-major
//   TN (wgrad,   dW = dy^T x): A M-major,  B N-major
// MN-major operands are loaded as 64-element-wide boxes (one 128-byte swizzle
// row per k) and described to the MMA as MN-major; no operand is transposed in
// memory. Skinny weight-gradient shapes are split along K; their partial sums
// are added to the fp32 gradient with atomics.
#include <cudaTypedefs.h>

#include <cstring>

#include "epilogue.cuh"
#include "tc_ptx.cuh"

namespace gpt2 {

namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;   // 16 KB
constexpr int B_BYTES = BN * BK * 2;   // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int MN_BOX_BYTES = 64 * BK * 2;       // one 64-wide MN-major box: 8 KB
constexpr int TMEM_COLS = 2 * BN;               // two accumulators
constexpr int EPI_BYTES = 32 * 1024;            // epilogue staging, split evenly among the epilogue warps

struct Ctl {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    uint32_t abort;
};

constexpr size_t SMEM_BYTES = (size_t)STAGES * STAGE_BYTES + EPI_BYTES + 1024 + sizeof(Ctl);

// Byte offset of 16-byte segment c of row r (0..31) in a warp's chunk buffer
// of ROWB-byte rows; the XOR spreads eight consecutive rows over all 32 banks,
// so both access patterns (a lane per row, and ROWB / 16 lanes per row) take the
// minimum four wavefronts per 512 bytes.
template <int ROWB>
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return ROWB == 128 ? r * 128 + ((c ^ (r & 7)) << 4) : r * 64 + ((c ^ ((r >> 1) & 3)) << 4);
}

struct Units {
    int tiles_m, tiles_n, splits, kb_total, kb_per_split;
    int m_fastest;   // walk m blocks fastest (B streamed once, A re-read) instead of n blocks
    __device__ __forceinline__ int count() const { return tiles_m * tiles_n * splits; }
    // unit -> (m block, n block, first and end k-block); the fast block index, then the
    // other, then split. The CTAs running at one time share the slow index's operand block.
    __device__ __forceinline__ void decode(int u, int& mb, int& nb, int& kb0, int& kb1) const {
        if (m_fastest) {
            mb = u % tiles_m;
            nb = (u / tiles_m) % tiles_n;
        } else {
            nb = u % tiles_n;
            mb = (u / tiles_n) % tiles_m;
        }
        const int s = u / (tiles_n * tiles_m);
        kb0 = s * kb_per_split;
        kb1 = min(kb_total, kb0 + kb_per_split);
    }
};

template <int KIND>
struct EpiTraits {
    static constexpr bool F32 = (KIND == EPI_BIAS_RESID || KIND == EPI_ACCUM_F32);   // fp32 result
    static constexpr bool WIDE = (KIND == EPI_BIAS_GELU);   // sixteen epilogue warps
    static constexpr int WARPS = WIDE ? 16 : 8;
    static constexpr int THREADS = 64 + 32 * WARPS;
    static constexpr int ROWB = WIDE ? 64 : 128;   // staged bytes per row and chunk
    static constexpr int SEGS = ROWB / 16;         // 16-byte segments per staged row = lanes per row when copying
    static constexpr int RPS = 32 / SEGS;          // rows per copy step
    static constexpr int EBUF = 32 * ROWB;         // staging per epilogue warp
    static constexpr int ES = F32 ? 4 : 2;         // element size
    static constexpr int CW = ROWB / ES;           // columns per chunk
    static constexpr int EPS = 16 / ES;            // elements per 16-byte segment
    static constexpr int WCOLS = BN / (WARPS / 4); // columns per warp and tile
    static constexpr bool HAS_IN = (KIND == EPI_BIAS_RESID || KIND == EPI_MUL);
    static constexpr bool HAS_BIAS = (KIND == EPI_BIAS || KIND == EPI_BIAS_GELU || KIND == EPI_BIAS_RESID);
    static constexpr int DEPTH = F32 ? 2 : 1;      // input chunks prefetched ahead (fp32 chunks are narrower)
};

// Start the coalesced loads of one input chunk (the residual, or the stored
// GELU derivative) into registers: SEGS lanes per row, RPS rows per step.
template <int KIND>
__device__ __forceinline__ void prefetch_in(const Epilogue& ep, uint4 (&pre)[EpiTraits<KIND>::SEGS], int row0,
                                            int col0, int M, int N) {
    using E = EpiTraits<KIND>;
    const int lane = threadIdx.x & 31;
    const int lrow = lane / E::SEGS, lseg = lane % E::SEGS;
    const char* src = KIND == EPI_BIAS_RESID ? reinterpret_cast<const char*>(ep.resid)
                                             : reinterpret_cast<const char*>(ep.aux);
#pragma unroll
    for (int st = 0; st < E::SEGS; ++st) {
        const int r = st * E::RPS + lrow;
        const int c = col0 + lseg * E::EPS;
        pre[st] = make_uint4(0, 0, 0, 0);
        if (row0 + r < M && c < N)
            pre[st] = *reinterpret_cast<const uint4*>(src + ((long long)(row0 + r) * ep.ldo + c) * E::ES);
    }
}

// One chunk of the epilogue for the calling warp: rows row0 .. row0+31 (lane =
// row of acc) by CW columns from col0. Results (and the prefetched residual /
// GELU' inputs, which have the same shape as the result) pass through the
// warp's shared-memory buffer, so global memory is read and written in
// ROWB-byte row segments, RPS rows per instruction; each lane updates its
// row's 16-byte segments in place in the buffer. If next_col0 >= 0, the input
// chunk at next_col0 is prefetched into `pre` while this chunk is computed.
template <int KIND>
__device__ __forceinline__ void epilogue_chunk(const Epilogue& ep, float* acc, int row0, int col0, int M, int N,
                                               uint8_t* buf, float4 bq, uint4 (&pre)[EpiTraits<KIND>::SEGS],
                                               int next_col0) {
    using E = EpiTraits<KIND>;
    constexpr bool F32 = E::F32;
    constexpr int EPS = E::EPS;
    constexpr int ES = E::ES;
    constexpr int kind = KIND;
    const int lane = threadIdx.x & 31;
    constexpr int ROWB = E::ROWB;
    const int lrow = lane / E::SEGS, lseg = lane % E::SEGS;   // copy pattern: SEGS lanes per row
    if (E::HAS_IN) {
#pragma unroll
        for (int st = 0; st < E::SEGS; ++st)
            *reinterpret_cast<uint4*>(buf + swz<ROWB>(st * E::RPS + lrow, lseg)) = pre[st];
        __syncwarp();
        if (next_col0 >= 0) prefetch_in<KIND>(ep, pre, row0, next_col0, M, N);
    }
    constexpr int npass = kind == EPI_BIAS_GELU ? 2 : 1;   // GELU: gelu'(u) (out2), then gelu(u) (out)
#pragma unroll
    for (int pass = 0; pass < npass; ++pass) {
#pragma unroll
        for (int c = 0; c < ROWB / 16; ++c) {
            float* x = acc + c * EPS;
            float in[EPS], b[EPS];
            if (E::HAS_IN) {
                if (F32) {
                    const float4 q = *reinterpret_cast<const float4*>(buf + swz<ROWB>(lane, c));
                    in[0] = q.x; in[1] = q.y; in[2] = q.z; in[3] = q.w;
                } else {
                    load8(reinterpret_cast<const bf16*>(buf + swz<ROWB>(lane, c)), in);
                }
            }
            if (E::HAS_BIAS && pass == 0) {   // the chunk's bias: column 4 l + i sits in lane l, component i
#pragma unroll
                for (int g = 0; g < EPS / 4; ++g) {
                    const int src = (c * EPS) / 4 + g;
                    b[4 * g] = __shfl_sync(0xffffffffu, bq.x, src);
                    b[4 * g + 1] = __shfl_sync(0xffffffffu, bq.y, src);
                    b[4 * g + 2] = __shfl_sync(0xffffffffu, bq.z, src);
                    b[4 * g + 3] = __shfl_sync(0xffffffffu, bq.w, src);
                }
            }
            float v[EPS];
            if (kind == EPI_BIAS_GELU && pass == 0) {
                // u = acc + bias rounded to bf16; gelu(u) kept in x for pass 1, gelu'(u) out now
#pragma unroll
                for (int j = 0; j < EPS; j += 2) {
                    const float2 u = __bfloat1622float2(__floats2bfloat162_rn(x[j] + b[j], x[j + 1] + b[j + 1]));
                    gelu_both_x2(u.x, u.y, x[j], x[j + 1], v[j], v[j + 1]);
                }
            } else {
#pragma unroll
            for (int j = 0; j < EPS; ++j) {
                switch (kind) {
                case EPI_BIAS: v[j] = x[j] + b[j]; break;
                case EPI_BIAS_GELU:
                    if (pass == 0) {   // u as rounded to bf16; keep gelu(u) for the second pass
                        float g;
                        gelu_fast_both(__bfloat162float(__float2bfloat16_rn(x[j] + b[j])), g, v[j]);
                        x[j] = g;
                    } else {
                        v[j] = x[j];
                    }
                    break;
                case EPI_BIAS_RESID: v[j] = in[j] + (x[j] + b[j]); break;
                case EPI_MUL: v[j] = x[j] * in[j]; break;
                default: v[j] = x[j]; break;
                }
            }
            }
            if (F32) {
                *reinterpret_cast<float4*>(buf + swz<ROWB>(lane, c)) = make_float4(v[0], v[1], v[2], v[3]);
            } else {
                store8(reinterpret_cast<bf16*>(buf + swz<ROWB>(lane, c)), v);
            }
        }
        __syncwarp();
        // whole rows out to global memory
        char* dst = reinterpret_cast<char*>((kind == EPI_BIAS_GELU && pass == 0) ? ep.out2 : ep.out);
#pragma unroll
        for (int st = 0; st < E::SEGS; ++st) {
            const int r = st * E::RPS + lrow;
            const int c = col0 + lseg * EPS;
            if (row0 + r < M && c < N) {
                const uint4 q = *reinterpret_cast<const uint4*>(buf + swz<ROWB>(r, lseg));
                char* gp = dst + ((long long)(row0 + r) * ep.ldo + c) * ES;
                if (F32 && kind == EPI_ACCUM_F32) {
                    float4 a = *reinterpret_cast<const float4*>(&q);
                    if (ep.split_atomic) {
                        atomicAdd(reinterpret_cast<float4*>(gp), a);
                    } else {
                        if (ep.beta != 0.f) {
                            const float4 o = *reinterpret_cast<const float4*>(gp);
                            a.x += ep.beta * o.x; a.y += ep.beta * o.y; a.z += ep.beta * o.z; a.w += ep.beta * o.w;
                        }
                        *reinterpret_cast<float4*>(gp) = a;
                    }
                } else {
                    *reinterpret_cast<uint4*>(gp) = q;
                }
            }
        }
        if (kind == EPI_MUL && ep.colsum_part) {
            // column sums of the warp's 32 rows: lane l < 16 = columns 2 l, 2 l + 1 of the chunk
            if (lane < E::CW / 2) {
                float s0 = 0.f, s1 = 0.f;
                const int rmax = M - row0;
#pragma unroll
                for (int r = 0; r < 32; ++r) {
                    if (r < rmax) {
                        const uint32_t w2 =
                            *reinterpret_cast<const uint32_t*>(buf + swz<ROWB>(r, lane >> 2) + (lane & 3) * 4);
                        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w2));
                        s0 += f.x;
                        s1 += f.y;
                    }
                }
                const int c = col0 + 2 * lane;
                if (c < N)
                    *reinterpret_cast<float2*>(ep.colsum_part + (long long)(row0 >> 5) * N + c) = make_float2(s0, s1);
            }
        }
        __syncwarp();
    }
}

template <int A_MN, int B_MN, int KIND>
__global__ void __launch_bounds__(EpiTraits<KIND>::THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M, int N,
                   Units units, Epilogue ep, unsigned* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* epi_smem = smem + STAGES * STAGE_BYTES;
    Ctl* ctl = reinterpret_cast<Ctl*>(epi_smem + EPI_BYTES);
    volatile uint32_t* abort = &ctl->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_units = units.count();

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            tc::mbar_init(&ctl->full[s], 1);
            tc::mbar_init(&ctl->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(&ctl->acc_full[b], 1);
            tc::mbar_init(&ctl->acc_empty[b], EpiTraits<KIND>::WARPS);
        }
        tc::mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        tc::fence_barrier_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(&ctl->tmem_base, TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = ctl->tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------ producer
            tc::tma_prefetch_desc(&tmA);
            tc::tma_prefetch_desc(&tmB);
            uint32_t it = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
                int mb, nb, kb0, kb1;
                units.decode(u, mb, nb, kb0, kb1);
                const int m0 = mb * BM, n0 = nb * BN;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!tc::mbar_wait(&ctl->empty[s], ph ^ 1, abort, status)) { ok = false; break; }
                    tc::mbar_expect_tx(&ctl->full[s], STAGE_BYTES);
                    uint8_t* sa = smem + s * STAGE_BYTES;
                    uint8_t* sb = sa + A_BYTES;
                    const int k0 = kb * BK;
                    if (A_MN) {
                        tc::tma_load_2d(sa, &tmA, m0, k0, &ctl->full[s]);
                        tc::tma_load_2d(sa + MN_BOX_BYTES, &tmA, m0 + 64, k0, &ctl->full[s]);
                    } else {
                        tc::tma_load_2d(sa, &tmA, k0, m0, &ctl->full[s]);
                    }
                    if (B_MN) {
#pragma unroll
                        for (int c = 0; c < BN / 64; ++c)
                            tc::tma_load_2d(sb + c * MN_BOX_BYTES, &tmB, n0 + 64 * c, k0, &ctl->full[s]);
                    } else {
                        tc::tma_load_2d(sb, &tmB, k0, n0, &ctl->full[s]);
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ----------------------------------------------------- MMA issue
            constexpr uint32_t idesc = tc::idesc_bf16_f32(BM, BN, A_MN, B_MN);
            uint32_t it = 0, acc_it = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++acc_it) {
                int mb, nb, kb0, kb1;
                units.decode(u, mb, nb, kb0, kb1);
                const uint32_t ab = acc_it & 1, aph = (acc_it >> 1) & 1;
                if (!tc::mbar_wait(&ctl->acc_empty[ab], aph ^ 1, abort, status)) break;
                tc::fence_after_sync();
                const uint32_t d_tmem = tmem + ab * BN;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!tc::mbar_wait(&ctl->full[s], ph, abort, status)) { ok = false; break; }
                    tc::fence_after_sync();
                    const uint32_t a_base = tc::smem_u32(smem + s * STAGE_BYTES);
                    const uint32_t b_base = a_base + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        // K-major: +32 bytes per 16-element k step inside the swizzle row;
                        // MN-major: +16 rows of 128 bytes.
                        const uint64_t da = A_MN ? tc::smem_desc_sw128(a_base + kk * 2048, MN_BOX_BYTES, 1024)
                                                 : tc::smem_desc_sw128(a_base + kk * 32, 16, 1024);
                        const uint64_t db = B_MN ? tc::smem_desc_sw128(b_base + kk * 2048, MN_BOX_BYTES, 1024)
                                                 : tc::smem_desc_sw128(b_base + kk * 32, 16, 1024);
                        tc::mma_bf16(d_tmem, da, db, idesc, (kb > kb0 || kk > 0) ? 1u : 0u);
                    }
                    tc::mma_commit(&ctl->empty[s]);   // stage free once these MMAs finish
                }
                tc::mma_commit(&ctl->acc_full[ab]);    // accumulator ready for the epilogue
            }
            // every MMA issued by this thread has completed once `drain` fires; this
            // wait ignores an abort (it must not free TMEM under running MMAs) but is
            // still bounded in time
            volatile uint32_t no_abort = 0;
            tc::mma_commit(&ctl->drain);
            tc::mbar_wait(&ctl->drain, 0, &no_abort, status);
        }
    } else {
        // ---------------------------------------------------------- epilogue
        using E = EpiTraits<KIND>;
        const int ew = warp - 2;                 // 0 .. E::WARPS - 1
        const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
        const int col_q = ew >> 2;               // columns [col_q * WCOLS, col_q * WCOLS + WCOLS)
        uint8_t* buf = epi_smem + ew * E::EBUF;
        constexpr int CW = E::CW;
        constexpr int NCH = E::WCOLS / CW;       // chunks per warp and tile
        uint4 pre[E::DEPTH][E::SEGS];            // input chunks in flight (ring)
        // the bias of one chunk: lane l < CW / 4 holds columns 4 l .. 4 l + 3 (zero past N),
        // loaded one chunk ahead; the chunk's lanes read it with shuffles
        auto load_bias = [&](int col0) {
            float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
            if (E::HAS_BIAS && lane < CW / 4 && col0 + 4 * lane < N)
                q = *reinterpret_cast<const float4*>(ep.bias + col0 + 4 * lane);
            return q;
        };
        uint32_t acc_it = 0;
        for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++acc_it) {
            int mb, nb, kb0, kb1;
            units.decode(u, mb, nb, kb0, kb1);
            const uint32_t ab = acc_it & 1, aph = (acc_it >> 1) & 1;
            const int row0 = mb * BM + quarter * 32;
            const int cbase = col_q * E::WCOLS;
            float4 bq = load_bias(nb * BN + cbase);
            // the first input chunks of this tile are requested before waiting for the accumulator
            if (E::HAS_IN && row0 < M) {
#pragma unroll
                for (int d = 0; d < E::DEPTH; ++d)
                    if (d < NCH) prefetch_in<KIND>(ep, pre[d], row0, nb * BN + cbase + d * CW, M, N);
            }
            uint32_t ok = 0;
            if (lane == 0) ok = tc::mbar_wait(&ctl->acc_full[ab], aph, abort, status) ? 1u : 0u;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc::fence_after_sync();
            const uint32_t taddr = tmem + ab * BN + cbase + ((uint32_t)(quarter * 32) << 16);
#pragma unroll
            for (int ci = 0; ci < NCH; ++ci) {
                const int c = ci * CW;
                const int col0 = nb * BN + cbase + c;
                if (col0 >= N) break;
                const float4 bcur = bq;
                if (E::HAS_BIAS && ci + 1 < NCH) bq = load_bias(col0 + CW);
                float acc[CW];
                if (CW == 64) {
                    tc::tmem_ld_32x32b_x32(taddr + (uint32_t)c, acc);
                    tc::tmem_ld_32x32b_x32(taddr + (uint32_t)c + 32, acc + 32);
                } else if (CW == 32) {
                    tc::tmem_ld_32x32b_x32(taddr + (uint32_t)c, acc);
                } else {
                    tc::tmem_ld_32x32b_x16(taddr + (uint32_t)c, acc);
                }
                const int nc = c + E::DEPTH * CW;     // chunk whose input this buffer prefetches next
                const int next = (nc < E::WCOLS && nb * BN + cbase + nc < N) ? nb * BN + cbase + nc : -1;
                if (row0 < M) epilogue_chunk<KIND>(ep, acc, row0, col0, M, N, buf, bcur, pre[ci % E::DEPTH], next);
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&ctl->acc_empty[ab]);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tmem, TMEM_COLS);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// Row-major matrix [rows][cols] with row stride ld (elements); box = box_cols
// (inner) x box_rows.
bool make_map_t(CUtensorMap* m, const void* ptr, bool f32, long long rows, long long cols, long long ld,
                int box_cols, int box_rows, CUtensorMapSwizzle sw) {
    auto fn = encode_fn();
    if (!fn) return false;
    const int es = f32 ? 4 : 2;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ld * es};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                    const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Operand map: bf16 [rows][cols], 128-byte swizzle, 64-element inner box.
bool make_map(CUtensorMap* m, const bf16* ptr, long long rows, long long cols, int box_cols, int box_rows) {
    return make_map_t(m, ptr, false, rows, cols, cols, box_cols, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

int g_num_sms = 0;

template <int A_MN, int B_MN, int KIND>
void launch_kernel(dim3 grid, cudaStream_t stream, const CUtensorMap& ta, const CUtensorMap& tb, int M, int N,
                   const Units& u, const Epilogue& ep, unsigned* status) {
    static bool configured = false;
    if (!configured) {
        cudaFuncSetAttribute(gemm_tc_kernel<A_MN, B_MN, KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_BYTES);
        configured = true;
    }
    gemm_tc_kernel<A_MN, B_MN, KIND><<<grid, EpiTraits<KIND>::THREADS, SMEM_BYTES, stream>>>(ta, tb, M, N, u, ep,
                                                                                             status);
}

template <int A_MN, int B_MN>
bool launch_variant(const Ctx& ctx, const CUtensorMap& ta, const CUtensorMap& tb, int M, int N, int K,
                    Epilogue ep) {
    if (g_num_sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (g_num_sms <= 0) g_num_sms = 148;
    }
    Units u;
    u.tiles_m = ceil_div(M, BM);
    u.tiles_n = ceil_div(N, BN);
    u.kb_total = ceil_div(K, BK);
    u.splits = 1;
    const int tiles = u.tiles_m * u.tiles_n;
    // Split K when the output has too few tiles to fill the GPU and the epilogue
    // accumulates into fp32 (partials are then added with atomics). Every extra
    // split adds a full tile of fp32 atomics, so one wave of units when that
    // fills at least 85% of the SMs, else about two waves.
    if (ep.kind == EPI_ACCUM_F32 && ep.beta == 1.f && tiles < g_num_sms) {
        int s = g_num_sms / tiles;
        if (tiles * s * 100 < 85 * g_num_sms) s = (2 * g_num_sms + tiles / 2) / tiles;
        s = min(s, max(1, u.kb_total / 8));
        u.splits = max(1, s);
    }
    u.kb_per_split = ceil_div(u.kb_total, u.splits);
    u.splits = ceil_div(u.kb_total, u.kb_per_split);
    if (u.splits > 1) ep.split_atomic = 1;
    // The operand indexed by the fast block is re-read once per slow block: for unsplit GEMMs
    // make it the smaller one, which stays in L2 (the lm_head forward: 25 MB of activations
    // re-read, 77 MB of wte streamed once).
    u.m_fastest = (u.splits == 1 && (long long)M * K < (long long)N * K) ? 1 : 0;
    const int n_units = tiles * u.splits;
    const dim3 grid(min(n_units, g_num_sms));
    switch (ep.kind) {
    case EPI_STORE: launch_kernel<A_MN, B_MN, EPI_STORE>(grid, ctx.stream, ta, tb, M, N, u, ep, ctx.status); break;
    case EPI_BIAS: launch_kernel<A_MN, B_MN, EPI_BIAS>(grid, ctx.stream, ta, tb, M, N, u, ep, ctx.status); break;
    case EPI_BIAS_GELU:
        launch_kernel<A_MN, B_MN, EPI_BIAS_GELU>(grid, ctx.stream, ta, tb, M, N, u, ep, ctx.status);
        break;
    case EPI_BIAS_RESID:
        launch_kernel<A_MN, B_MN, EPI_BIAS_RESID>(grid, ctx.stream, ta, tb, M, N, u, ep, ctx.status);
        break;
    case EPI_MUL: launch_kernel<A_MN, B_MN, EPI_MUL>(grid, ctx.stream, ta, tb, M, N, u, ep, ctx.status); break;
    case EPI_ACCUM_F32:
        launch_kernel<A_MN, B_MN, EPI_ACCUM_F32>(grid, ctx.stream, ta, tb, M, N, u, ep, ctx.status);
        break;
    default: return false;
    }
    return true;
}

}  // namespace

bool gemm_tc_supported(GemmLayout layout, int M, int N, int K) {
    if (M < 1 || N < 1 || K < 1) return false;
    if (K % 8 != 0 || N % 8 != 0) return false;            // 16-byte row strides
    if (layout == GEMM_TN && M % 8 != 0) return false;      // A stored [K][M]
    return encode_fn() != nullptr;
}

bool launch_gemm_tc(const Ctx& ctx, GemmLayout layout, const bf16* A, const bf16* B, int M, int N, int K,
                    const Epilogue& ep) {
    CUtensorMap ta, tb;
    bool ok;
    switch (layout) {
    case GEMM_NT:   // A [M][K], B [N][K]
        ok = make_map(&ta, A, M, K, 64, BM) && make_map(&tb, B, N, K, 64, BN);
        if (ok) ok = launch_variant<0, 0>(ctx, ta, tb, M, N, K, ep);
        break;
    case GEMM_NN:   // A [M][K], B [K][N]
        ok = make_map(&ta, A, M, K, 64, BM) && make_map(&tb, B, K, N, 64, BK);
        if (ok) ok = launch_variant<0, 1>(ctx, ta, tb, M, N, K, ep);
        break;
    default:        // GEMM_TN: A [K][M], B [K][N]
        ok = make_map(&ta, A, K, M, 64, BK) && make_map(&tb, B, K, N, 64, BK);
        if (ok) ok = launch_variant<1, 1>(ctx, ta, tb, M, N, K, ep);
        break;
    }
    if (ok) ++*ctx.launches;
    return ok;
}

}  // namespace gpt2
