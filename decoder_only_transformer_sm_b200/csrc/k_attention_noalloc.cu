// Attention backward for callers that cannot allocate device memory.
//
// gpt2k_attention_bwd needs a scratch vector of B*H*T floats (the per-row
// D = rowsum(dout * out) of the softmax backward), which its caller must
// allocate. Some callers cannot call cudaMalloc: code that runs inside a
// framework whose caching allocator owns all device memory (a raw cudaMalloc
// bypasses the pool, can fail when the pool holds the memory, and fragments
// it), and latency-critical loops where cudaMalloc's implicit device
// synchronisation is not allowed. gpt2k_attention_bwd_noalloc takes the same
// inputs and outputs but no workspace: its scratch is the fixed array below,
// which lives in the library's device image, so every GPU that loads the
// library holds it (1 MiB) until the process exits.
//
// Host code cannot pass the array's name to a kernel (on the host the name is
// only a stand-in, not a device address). The first call on each device, with
// that device current, asks the runtime for the array's device address with
// cudaGetSymbolAddress and caches it per device; later calls reuse it.
//
// All calls share the one array and it keeps the last call's contents. The
// backward's pre-pass writes every element of D that the later passes read, so
// nothing has to be cleared between calls. Calls that overlap on the GPU (for
// instance on two streams at once) race on the array and must not be issued.
#include <mutex>

#include "gpt2_kernels.h"
#include "kernels.cuh"

using namespace gpt2;

namespace gpt2 {
int set_error(int code, const char* msg);   // defined in gpt2_api.cu
}

namespace {

constexpr long long NOALLOC_MAX_ROWS = 262144;   // B*H*T limit: 1 MiB of fp32 scratch
constexpr int MAX_DEVICES = 64;

static __device__ __align__(256) float g_attn_bwd_scratch[NOALLOC_MAX_ROWS];

std::mutex g_scratch_mu;
float* g_scratch_ptr[MAX_DEVICES] = {};

// Device address of g_attn_bwd_scratch on the current device (set up once per device).
int scratch_address(float** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_error(GPT2_ERR_CUDA, cudaGetErrorString(e));
    if (dev < 0 || dev >= MAX_DEVICES) return set_error(GPT2_ERR_INVALID_ARG, "device ordinal out of range");
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_attn_bwd_scratch);
        if (e != cudaSuccess || !p) {
            cudaGetLastError();
            return set_error(GPT2_ERR_CUDA, "cudaGetSymbolAddress of the attention scratch failed");
        }
        g_scratch_ptr[dev] = static_cast<float*>(p);
    }
    *out = g_scratch_ptr[dev];
    return GPT2_OK;
}

}  // namespace

extern "C" int gpt2k_attention_bwd_noalloc(int dtype, const void* qkv, const void* out, const void* dout,
                                           const float* lse, void* dqkv, int B, int T, int H, int hd, int engine,
                                           uint32_t* status_dev, void* stream) {
    if (dtype != GPT2K_F32 && dtype != GPT2K_BF16) return set_error(GPT2_ERR_INVALID_ARG, "unknown dtype");
    if (B < 1 || T < 1 || H < 1) return set_error(GPT2_ERR_INVALID_ARG, "B, T, H must be >= 1");
    if (hd != 32 && hd != 64) return set_error(GPT2_ERR_INVALID_ARG, "head width must be 32 or 64");
    if (engine != 0) return set_error(GPT2_ERR_INVALID_ARG, "unknown attention engine");
    if (!qkv || !out || !dout || !lse || !dqkv || !status_dev)
        return set_error(GPT2_ERR_INVALID_ARG, "NULL operand");
    if ((long long)B * H * T > NOALLOC_MAX_ROWS)
        return set_error(GPT2_ERR_INVALID_ARG,
                         "B*H*T exceeds 262144, the row limit of the no-allocation attention backward; "
                         "use gpt2k_attention_bwd with a caller-allocated workspace");
    float* scratch = nullptr;
    int rc = scratch_address(&scratch);
    if (rc) return rc;
    long long launches = 0;
    Ctx c;
    c.stream = (cudaStream_t)stream;
    c.status = status_dev;
    c.launches = &launches;
    c.num_sms = 148;
    if (dtype == GPT2K_F32)
        launch_attention_bwd_simt<float>(c, (const float*)qkv, (const float*)out, (const float*)dout, lse, scratch,
                                         (float*)dqkv, B, T, H, hd);
    else
        launch_attention_bwd_simt<bf16>(c, (const bf16*)qkv, (const bf16*)out, (const bf16*)dout, lse, scratch,
                                        (bf16*)dqkv, B, T, H, hd);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return set_error(GPT2_ERR_CUDA, cudaGetErrorString(err));
    return GPT2_OK;
}
