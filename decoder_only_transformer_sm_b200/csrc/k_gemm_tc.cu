// Tensor-core GEMM for sm_100a: TMA loads into a multi-stage shared-memory
// ring, tcgen05.mma (kind::f16, bf16 operands) issued by one thread into an
// fp32 accumulator in tensor memory, and an epilogue that reads the
// accumulator with tcgen05.ld and applies the fused bias / GELU / residual /
// dGELU / fp32-accumulate step while storing.
//
// All three operand layouts of the training step run on the same kernel:
//   NT (forward, y = x W^T):   A K-major,  B K-major
//   NN (dgrad,   dx = dy W):   A K-major,  B N-major
//   TN (wgrad,   dW = dy^T x): A M-major,  B N-major
// MN-major operands are loaded as 64-element-wide boxes (one 128-byte swizzle
// row per k) and described to the MMA as MN-major; no operand is transposed
// in memory.
//
// Warp roles (192 threads): warp 0 = TMA producer, warp 1 = TMEM owner and
// MMA issuer, warps 2..5 = epilogue (TMEM lane quarter = warp % 4).
#include <cudaTypedefs.h>

#include "epilogue.cuh"
#include "tc_ptx.cuh"

namespace gpt2 {

namespace {

constexpr int BM = 128, BN = 128, BK = 64, STAGES = 3;   // 2 CTAs per SM
constexpr int A_BYTES = BM * BK * 2;   // 16 KB
constexpr int B_BYTES = BN * BK * 2;   // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr int MN_BOX_BYTES = 64 * BK * 2;   // one 64-wide MN-major box: 8 KB

struct Ctl {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t accum;
    uint32_t tmem_base;
    uint32_t abort;
};

constexpr size_t SMEM_BYTES = (size_t)STAGES * STAGE_BYTES + 1024 + sizeof(Ctl);

template <int A_MN, int B_MN>
__global__ void __launch_bounds__(THREADS, 2)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M, int N,
                   int K, Epilogue ep, unsigned* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctl* ctl = reinterpret_cast<Ctl*>(smem + STAGES * STAGE_BYTES);
    volatile uint32_t* abort = &ctl->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    const int num_kb = (K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            tc::mbar_init(&ctl->full[s], 1);
            tc::mbar_init(&ctl->empty[s], 1);
        }
        tc::mbar_init(&ctl->accum, 1);
        ctl->abort = 0;
        tc::fence_barrier_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(&ctl->tmem_base, BN);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = ctl->tmem_base;

    if (warp == 0 && lane == 0) {
        // ---------------------------------------------------------- producer
        tc::tma_prefetch_desc(&tmA);
        tc::tma_prefetch_desc(&tmB);
        for (int kb = 0; kb < num_kb; ++kb) {
            const int s = kb % STAGES;
            const uint32_t ph = (kb / STAGES) & 1;
            if (!tc::mbar_wait(&ctl->empty[s], ph ^ 1, abort, status)) break;
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
                tc::tma_load_2d(sb, &tmB, n0, k0, &ctl->full[s]);
                tc::tma_load_2d(sb + MN_BOX_BYTES, &tmB, n0 + 64, k0, &ctl->full[s]);
            } else {
                tc::tma_load_2d(sb, &tmB, k0, n0, &ctl->full[s]);
            }
        }
    } else if (warp == 1 && lane == 0) {
        // --------------------------------------------------------- MMA issue
        constexpr uint32_t idesc = tc::idesc_bf16_f32(BM, BN, A_MN, B_MN);
        for (int kb = 0; kb < num_kb; ++kb) {
            const int s = kb % STAGES;
            const uint32_t ph = (kb / STAGES) & 1;
            if (!tc::mbar_wait(&ctl->full[s], ph, abort, status)) break;
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
                tc::mma_bf16(tmem, da, db, idesc, (kb | kk) != 0 ? 1u : 0u);
            }
            tc::mma_commit(&ctl->empty[s]);   // stage free once these MMAs finish
        }
        tc::mma_commit(&ctl->accum);          // accumulator complete (also after an abort)
    } else if (warp >= 2) {
        // ---------------------------------------------------------- epilogue
        uint32_t ok = 0;
        if (lane == 0) ok = tc::mbar_wait(&ctl->accum, 0, abort, status) ? 1u : 0u;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (ok) {
            tc::fence_after_sync();
            const int quarter = warp & 3;
            const int row = m0 + quarter * 32 + lane;
#pragma unroll 1
            for (int c = 0; c < BN; c += 32) {
                float acc[32];
                tc::tmem_ld_32x32b_x32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)c, acc);
                if (row < M && n0 + c < N) epilogue_run<bf16, 32>(ep, row, n0 + c, N, acc);
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tmem, BN);
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

// Row-major bf16 matrix [rows][cols]; box = box_cols (inner, 64 = 128 B) x box_rows.
bool make_map(CUtensorMap* m, const bf16* ptr, long long rows, long long cols, int box_cols, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<bf16*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int A_MN, int B_MN>
void launch_variant(const Ctx& ctx, const CUtensorMap& ta, const CUtensorMap& tb, int M, int N, int K,
                    const Epilogue& ep) {
    static bool configured = false;
    if (!configured) {
        cudaFuncSetAttribute(gemm_tc_kernel<A_MN, B_MN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_BYTES);
        configured = true;
    }
    dim3 grid(ceil_div(N, BN), ceil_div(M, BM));
    gemm_tc_kernel<A_MN, B_MN><<<grid, THREADS, SMEM_BYTES, ctx.stream>>>(ta, tb, M, N, K, ep, ctx.status);
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
        if (ok) launch_variant<0, 0>(ctx, ta, tb, M, N, K, ep);
        break;
    case GEMM_NN:   // A [M][K], B [K][N]
        ok = make_map(&ta, A, M, K, 64, BM) && make_map(&tb, B, K, N, 64, BK);
        if (ok) launch_variant<0, 1>(ctx, ta, tb, M, N, K, ep);
        break;
    default:        // GEMM_TN: A [K][M], B [K][N]
        ok = make_map(&ta, A, K, M, 64, BK) && make_map(&tb, B, K, N, 64, BK);
        if (ok) launch_variant<1, 1>(ctx, ta, tb, M, N, K, ep);
        break;
    }
    if (ok) ++*ctx.launches;
    return ok;
}

}  // namespace gpt2
