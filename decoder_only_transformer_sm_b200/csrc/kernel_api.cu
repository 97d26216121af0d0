// Kernel-level C ABI (gpt2_kernels.h): single operations on caller-owned
// device buffers.
#include <string>

#include "gpt2_kernels.h"
#include "kernels.cuh"

using namespace gpt2;

namespace gpt2 {
int set_error(int code, const char* msg);   // defined in gpt2_api.cu
}

extern "C" int gpt2k_matmul_bf16(int layout, const void* A, const void* B, int M, int N, int K, int epilogue,
                                 void* out, int64_t ldo, void* out2, const float* bias, const float* resid,
                                 const void* aux, float* colsum_part, float beta, int engine,
                                 uint32_t* status_dev, void* stream) {
    if (layout < GPT2K_NT || layout > GPT2K_TN) return set_error(GPT2_ERR_INVALID_ARG, "unknown layout");
    if (epilogue < GPT2K_EPI_STORE || epilogue > GPT2K_EPI_ACCUM_F32)
        return set_error(GPT2_ERR_INVALID_ARG, "unknown epilogue");
    if (M < 1 || N < 1 || K < 1 || ldo < N) return set_error(GPT2_ERR_INVALID_ARG, "bad sizes");
    if (!A || !B || !out || !status_dev) return set_error(GPT2_ERR_INVALID_ARG, "NULL operand");
    const bool needs_bias = epilogue == GPT2K_EPI_BIAS || epilogue == GPT2K_EPI_BIAS_GELU ||
                            epilogue == GPT2K_EPI_BIAS_RESID;
    if ((needs_bias && !bias) || (epilogue == GPT2K_EPI_BIAS_GELU && !out2) ||
        (epilogue == GPT2K_EPI_BIAS_RESID && !resid) || (epilogue == GPT2K_EPI_MUL && !aux))
        return set_error(GPT2_ERR_INVALID_ARG, "epilogue operand missing");
    if (colsum_part && (epilogue != GPT2K_EPI_MUL || engine != 1))
        return set_error(GPT2_ERR_INVALID_ARG, "column sums come only with the tensor-core GPT2K_EPI_MUL epilogue");
    long long launches = 0;
    Ctx c;
    c.stream = (cudaStream_t)stream;
    c.status = status_dev;
    c.launches = &launches;
    c.num_sms = 148;
    Epilogue e;
    e.kind = epilogue;
    e.out = out;
    e.ldo = ldo;
    e.out2 = out2;
    e.bias = bias;
    e.resid = resid;
    e.aux = aux;
    e.colsum_part = colsum_part;
    e.beta = beta;
    const GemmLayout L = (GemmLayout)layout;
    if (engine == 1) {
        if (!gemm_tc_supported(L, M, N, K))
            return set_error(GPT2_ERR_INVALID_ARG, "shape not supported by the tensor-core GEMM");
        if (ldo % 8 != 0) return set_error(GPT2_ERR_INVALID_ARG, "the tensor-core GEMM needs ldo % 8 == 0");
        if (epilogue == GPT2K_EPI_ACCUM_F32 && beta != 0.f && beta != 1.f)
            return set_error(GPT2_ERR_INVALID_ARG, "the tensor-core GEMM accumulates with beta 0 or 1");
        if (!launch_gemm_tc(c, L, (const bf16*)A, (const bf16*)B, M, N, K, e))
            return set_error(GPT2_ERR_CUDA, "tensor-map encoding failed");
    } else {
        launch_gemm_simt<bf16>(c, L, (const bf16*)A, (const bf16*)B, M, N, K, e);
    }
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return set_error(GPT2_ERR_CUDA, cudaGetErrorString(err));
    return GPT2_OK;
}

namespace {
int check_attention_args(int dtype, int B, int T, int H, int hd, int engine, const void* a, const void* b,
                         const void* c, const uint32_t* status) {
    if (dtype != GPT2K_F32 && dtype != GPT2K_BF16) return set_error(GPT2_ERR_INVALID_ARG, "unknown dtype");
    if (B < 1 || T < 1 || H < 1) return set_error(GPT2_ERR_INVALID_ARG, "B, T, H must be >= 1");
    if (hd != 32 && hd != 64) return set_error(GPT2_ERR_INVALID_ARG, "head width must be 32 or 64");
    if (engine < 0 || engine > 2) return set_error(GPT2_ERR_INVALID_ARG, "unknown attention engine");
    if (engine >= 1 && dtype != GPT2K_BF16)
        return set_error(GPT2_ERR_INVALID_ARG, "the tensor-core attention engines take bf16 operands");
    if (engine == 2 && hd != 64)
        return set_error(GPT2_ERR_INVALID_ARG, "the tcgen05 attention engine needs head width 64");
    if (!a || !b || !c || !status) return set_error(GPT2_ERR_INVALID_ARG, "NULL operand");
    return GPT2_OK;
}

Ctx kctx(void* stream, uint32_t* status, long long* launches) {
    Ctx c;
    c.stream = (cudaStream_t)stream;
    c.status = status;
    c.launches = launches;
    c.num_sms = 148;
    return c;
}
}  // namespace

extern "C" int gpt2k_attention_fwd(int dtype, const void* qkv, void* out, float* lse, int B, int T, int H, int hd,
                                   int engine, uint32_t* status_dev, void* stream) {
    int rc = check_attention_args(dtype, B, T, H, hd, engine, qkv, out, lse, status_dev);
    if (rc) return rc;
    long long launches = 0;
    Ctx c = kctx(stream, status_dev, &launches);
    if (engine == 2) {
        if (!launch_attention_fwd_tc(c, (const bf16*)qkv, (bf16*)out, lse, B, T, H))
            return set_error(GPT2_ERR_CUDA, "tensor-map encoding failed");
    } else if (engine == 1)
        launch_attention_fwd_mma(c, (const bf16*)qkv, (bf16*)out, lse, B, T, H, hd);
    else if (dtype == GPT2K_F32)
        launch_attention_fwd_simt<float>(c, (const float*)qkv, (float*)out, lse, B, T, H, hd);
    else
        launch_attention_fwd_simt<bf16>(c, (const bf16*)qkv, (bf16*)out, lse, B, T, H, hd);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return set_error(GPT2_ERR_CUDA, cudaGetErrorString(err));
    return GPT2_OK;
}

namespace {
// engine 2 workspace: [D: B*H*T floats, padded to 64][dQ accumulator: B*T*C floats][work counter: 64]
long long attention_bwd_dq_offset(int B, int T, int H) { return ((long long)B * H * T + 63) / 64 * 64; }
long long attention_bwd_work_offset(int B, int T, int H, int hd) {
    return attention_bwd_dq_offset(B, T, H) + ((long long)B * T * H * hd + 63) / 64 * 64;
}
}  // namespace

extern "C" int gpt2k_attention_bwd_workspace(int B, int T, int H, int hd, int engine, int64_t* floats) {
    if (!floats) return set_error(GPT2_ERR_INVALID_ARG, "NULL argument");
    if (B < 1 || T < 1 || H < 1 || (hd != 32 && hd != 64) || engine < 0 || engine > 2)
        return set_error(GPT2_ERR_INVALID_ARG, "bad size, head width or engine");
    *floats = engine == 2 ? attention_bwd_work_offset(B, T, H, hd) + 64 : (long long)B * H * T;
    return GPT2_OK;
}

extern "C" int gpt2k_attention_bwd(int dtype, const void* qkv, const void* out, const void* dout, const float* lse,
                                   void* dqkv, int B, int T, int H, int hd, float* workspace_dev,
                                   float* colsum_part, int engine, uint32_t* status_dev, void* stream) {
    int rc = check_attention_args(dtype, B, T, H, hd, engine, qkv, out, dout, status_dev);
    if (rc) return rc;
    if (!lse || !dqkv || !workspace_dev) return set_error(GPT2_ERR_INVALID_ARG, "NULL operand");
    if (colsum_part && engine != 2)
        return set_error(GPT2_ERR_INVALID_ARG, "column sums come only with the tcgen05 attention backward");
    long long launches = 0;
    Ctx c = kctx(stream, status_dev, &launches);
    if (engine == 2) {
        if (!launch_attention_bwd_tc(c, (const bf16*)qkv, (const bf16*)out, (const bf16*)dout, lse, workspace_dev,
                                     workspace_dev + attention_bwd_dq_offset(B, T, H),
                                     (int*)(workspace_dev + attention_bwd_work_offset(B, T, H, hd)), (bf16*)dqkv, B,
                                     T, H, colsum_part))
            return set_error(GPT2_ERR_CUDA, "tensor-map encoding failed");
    } else if (engine == 1)
        launch_attention_bwd_mma(c, (const bf16*)qkv, (const bf16*)out, (const bf16*)dout, lse, workspace_dev,
                                 (bf16*)dqkv, B, T, H, hd);
    else if (dtype == GPT2K_F32)
        launch_attention_bwd_simt<float>(c, (const float*)qkv, (const float*)out, (const float*)dout, lse,
                                         workspace_dev, (float*)dqkv, B, T, H, hd);
    else
        launch_attention_bwd_simt<bf16>(c, (const bf16*)qkv, (const bf16*)out, (const bf16*)dout, lse,
                                        workspace_dev, (bf16*)dqkv, B, T, H, hd);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return set_error(GPT2_ERR_CUDA, cudaGetErrorString(err));
    return GPT2_OK;
}

extern "C" int gpt2k_attention_decode(int dtype, const void* cache, void* out, int B, int H, int hd, int Tc, int n,
                                      float* workspace_dev, uint32_t* status_dev, void* stream) {
    if (dtype != GPT2K_F32 && dtype != GPT2K_BF16) return set_error(GPT2_ERR_INVALID_ARG, "unknown dtype");
    if (B < 1 || H < 1 || Tc < 1 || n < 1 || n > Tc)
        return set_error(GPT2_ERR_INVALID_ARG, "need B, H >= 1 and 1 <= n <= Tc");
    if (hd != 32 && hd != 64) return set_error(GPT2_ERR_INVALID_ARG, "head width must be 32 or 64");
    if ((H * hd) % 64 != 0) return set_error(GPT2_ERR_INVALID_ARG, "C = H * hd must be a multiple of 64");
    if (!cache || !out || !workspace_dev || !status_dev) return set_error(GPT2_ERR_INVALID_ARG, "NULL operand");
    long long launches = 0;
    Ctx c = kctx(stream, status_dev, &launches);
    if (dtype == GPT2K_F32)
        launch_attention_decode<float>(c, (const float*)cache, (float*)out, workspace_dev, B, H, hd, Tc, n);
    else
        launch_attention_decode<bf16>(c, (const bf16*)cache, (bf16*)out, workspace_dev, B, H, hd, Tc, n);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return set_error(GPT2_ERR_CUDA, cudaGetErrorString(err));
    return GPT2_OK;
}

extern "C" int gpt2k_sample(int dtype, const void* logits, int rows, int V, int64_t ld, float temperature,
                            int top_k, const float* u_dev, int32_t* next_dev, uint32_t* status_dev, void* stream) {
    if (dtype != GPT2K_F32 && dtype != GPT2K_BF16) return set_error(GPT2_ERR_INVALID_ARG, "unknown dtype");
    if (rows < 1 || V < 1 || ld < V) return set_error(GPT2_ERR_INVALID_ARG, "need rows, V >= 1 and ld >= V");
    if (!logits || !u_dev || !next_dev || !status_dev) return set_error(GPT2_ERR_INVALID_ARG, "NULL operand");
    if (!(temperature > 0.f) || !(temperature < INFINITY))
        return set_error(GPT2_ERR_INVALID_ARG, "temperature must be finite and > 0");
    long long launches = 0;
    Ctx c = kctx(stream, status_dev, &launches);
    if (dtype == GPT2K_F32)
        launch_sample<float>(c, (const float*)logits, ld, rows, V, temperature, top_k, u_dev, next_dev, nullptr, 0, 0);
    else
        launch_sample<bf16>(c, (const bf16*)logits, ld, rows, V, temperature, top_k, u_dev, next_dev, nullptr, 0, 0);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return set_error(GPT2_ERR_CUDA, cudaGetErrorString(err));
    return GPT2_OK;
}

extern "C" int gpt2k_embedding_bwd_workspace(int B, int T, int C, int64_t* floats) {
    if (B < 1 || T < 1 || C < 1 || !floats) return set_error(GPT2_ERR_INVALID_ARG, "need B, T, C >= 1 and floats");
    *floats = (int64_t)embed_bwd_scratch_floats((long long)B * T, C);
    return GPT2_OK;
}

extern "C" int gpt2k_embedding_bwd(const int32_t* idx, const float* dx, int B, int T, int C, int V, float* dwte,
                                   float* dwpe, float* workspace_dev, uint32_t* status_dev, void* stream) {
    if (B < 1 || T < 1 || C < 1 || V < 1) return set_error(GPT2_ERR_INVALID_ARG, "need B, T, C, V >= 1");
    if (C % 4 != 0) return set_error(GPT2_ERR_INVALID_ARG, "C must be a multiple of 4");
    if (!idx || !dx || !dwte || !dwpe || !status_dev) return set_error(GPT2_ERR_INVALID_ARG, "NULL operand");
    long long launches = 0;
    Ctx c = kctx(stream, status_dev, &launches);
    launch_embed_bwd(c, idx, dx, B, T, C, V, dwte, dwpe, workspace_dev);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return set_error(GPT2_ERR_CUDA, cudaGetErrorString(err));
    return GPT2_OK;
}
