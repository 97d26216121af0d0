// Optimiser kernels: global gradient sum of squares, one multi-tensor clip +
// AdamW kernel over the flat parameter vector, the bf16 weight copy, and the
// on-device initial draw.
//
// Source definitions: "GPT-2 from Scratch", "Gradient clipping" (global L2 norm
// over all gradients, scaled so the norm is at most the threshold) and "AdamW,
// and weight decay on matrices only" (betas (0.9, 0.95), eps 1e-8, decay 0.1 on
// 2-D tensors); "Let's reproduce GPT-2 (124M)", "Matching GPT-3's optimization
// hyperparameters" (one fused kernel for all tensors). The AdamW form is the
// decoupled one of Loshchilov & Hutter with PyTorch's lr-scaled decay:
//   p <- p (1 - lr wd) - lr * (m / bc1) / (sqrt(v / bc2) + eps).
#include "kernels.cuh"

namespace gpt2 {

namespace {

__global__ void sumsq_kernel(const float* __restrict__ g, long long n, double* out) {
    float s = 0.f;
    const long long n4 = n / 4;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
        float4 v = reinterpret_cast<const float4*>(g)[i];
        s += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
    for (long long i = n4 * 4 + (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        s += g[i] * g[i];
    double d = warp_sum((double)s);
    __shared__ double part[32];
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = d;
    __syncthreads();
    if (threadIdx.x < 32) {
        d = (threadIdx.x < (blockDim.x >> 5)) ? part[threadIdx.x] : 0.0;
        d = warp_sum(d);
        if (threadIdx.x == 0) atomicAdd(out, d);
    }
}

__global__ void __launch_bounds__(256) adamw_kernel(const AdamChunk* __restrict__ chunks, float* __restrict__ p,
                                                    const float* __restrict__ g, float* __restrict__ m,
                                                    float* __restrict__ v, bf16* __restrict__ shadow,
                                                    const double* __restrict__ sumsq,
                                                    const double* __restrict__ loss_accum,
                                                    const unsigned* __restrict__ status, float lr, float clip,
                                                    float bc1, float bc2, float wd) {
    const double ss = *sumsq;
    const double loss = *loss_accum;
    // A step whose forward saw an out-of-range id, or whose kernels gave up a
    // bounded wait, is reported as an error by the host and must not move the
    // weights; neither must a non-finite loss or norm (reported as NONFINITE).
    if (*status & (STATUS_BAD_TOKEN | STATUS_TIMEOUT)) return;
    if (!isfinite(ss) || !isfinite(loss)) return;
    const float norm = (float)sqrt(ss);
    const float coef = fminf(1.f, clip / (norm + 1e-6f));
    const AdamChunk ch = chunks[blockIdx.x];
    const float dec = ch.decay ? (1.f - lr * wd) : 1.f;
    const float step = lr / bc1;
    const float rbc2 = 1.f / sqrtf(bc2);
    const long long s0 = ch.start;
    // chunks are multiples of 4 elements and start 16-byte aligned
    for (int i = threadIdx.x * 4; i < ch.count; i += blockDim.x * 4) {
        const long long k = s0 + i;
        float pp[4], gg[4], mm[4], vv[4];
        load4(p + k, pp); load4(g + k, gg); load4(m + k, mm); load4(v + k, vv);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float gc = gg[j] * coef;
            mm[j] = 0.9f * mm[j] + 0.1f * gc;
            vv[j] = 0.95f * vv[j] + 0.05f * gc * gc;
            const float denom = sqrtf(vv[j]) * rbc2 + 1e-8f;
            pp[j] = pp[j] * dec - step * (mm[j] / denom);
        }
        store4(p + k, pp); store4(m + k, mm); store4(v + k, vv);
        if (shadow) store4(shadow + k, pp);
    }
}

__global__ void to_bf16_kernel(const float* __restrict__ in, bf16* __restrict__ out, long long n) {
    const long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 4;
    if (i + 4 <= n) {
        float v[4];
        load4(in + i, v);
        store4(out + i, v);
    } else {
        for (long long k = i; k < n; ++k) out[k] = __float2bfloat16_rn(in[k]);
    }
}

// Philox4x32-10 (Salmon, Moraes, Dror, Shaw: "Parallel Random Numbers: As Easy
// as 1, 2, 3", SC'11): ten rounds of two 32x32->64 multiplies with a Weyl key
// schedule. Counter = (element quad index, stream id), key = seed.
struct U4 { unsigned x, y, z, w; };
__device__ __forceinline__ U4 philox4x32_10(U4 c, unsigned k0, unsigned k1) {
    const unsigned M0 = 0xD2511F53u, M1 = 0xCD9E8D57u, W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const unsigned hi0 = __umulhi(M0, c.x), lo0 = M0 * c.x;
        const unsigned hi1 = __umulhi(M1, c.z), lo1 = M1 * c.z;
        c = U4{hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0};
        k0 += W0;
        k1 += W1;
    }
    return c;
}

__device__ __forceinline__ float u01(unsigned x) {   // (0, 1]
    return ((float)(x >> 8) + 1.0f) * (1.0f / 16777216.0f);
}

// Box-Muller transform of two uniforms into two standard normals.
__global__ void fill_normal_kernel(float* p, long long n, float std, unsigned long long seed,
                                   unsigned long long stream_id) {
    const long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (q * 4 >= n) return;
    U4 c{(unsigned)q, (unsigned)(q >> 32), (unsigned)stream_id, (unsigned)(stream_id >> 32)};
    U4 r = philox4x32_10(c, (unsigned)seed, (unsigned)(seed >> 32));
    const float two_pi = 6.283185307179586f;
    float r1 = sqrtf(-2.f * logf(u01(r.x))), r2 = sqrtf(-2.f * logf(u01(r.z)));
    float z[4] = {r1 * cosf(two_pi * u01(r.y)), r1 * sinf(two_pi * u01(r.y)), r2 * cosf(two_pi * u01(r.w)),
                  r2 * sinf(two_pi * u01(r.w))};
    for (int j = 0; j < 4; ++j)
        if (q * 4 + j < n) p[q * 4 + j] = std * z[j];
}

__global__ void fill_const_kernel(float* p, long long n, float value) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) p[i] = value;
}

}  // namespace

void launch_sumsq(const Ctx& ctx, const float* g, long long n, double* out) {
    const int blocks = ctx.num_sms * 4;
    sumsq_kernel<<<blocks, 512, 0, ctx.stream>>>(g, n, out);
    ++*ctx.launches;
}

void launch_adamw(const Ctx& ctx, const AdamChunk* chunks, int n_chunks, float* p, const float* g, float* m,
                  float* v, bf16* shadow, const double* sumsq, const double* loss_accum, float lr, float clip,
                  float bc1, float bc2, float wd) {
    adamw_kernel<<<n_chunks, 256, 0, ctx.stream>>>(chunks, p, g, m, v, shadow, sumsq, loss_accum, ctx.status, lr,
                                                   clip, bc1, bc2, wd);
    ++*ctx.launches;
}

void launch_to_bf16(const Ctx& ctx, const float* in, bf16* out, long long n) {
    to_bf16_kernel<<<(unsigned)ceil_div_ll(ceil_div_ll(n, 4), 256), 256, 0, ctx.stream>>>(in, out, n);
    ++*ctx.launches;
}

void launch_fill_normal(const Ctx& ctx, float* p, long long n, float std, unsigned long long seed,
                        unsigned long long stream_id) {
    fill_normal_kernel<<<(unsigned)ceil_div_ll(ceil_div_ll(n, 4), 256), 256, 0, ctx.stream>>>(p, n, std, seed,
                                                                                              stream_id);
    ++*ctx.launches;
}

void launch_fill_const(const Ctx& ctx, float* p, long long n, float value) {
    fill_const_kernel<<<(unsigned)ceil_div_ll(n, 256), 256, 0, ctx.stream>>>(p, n, value);
    ++*ctx.launches;
}

}  // namespace gpt2
