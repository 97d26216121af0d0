// Shared device helpers of the CUDA path: types, conversions, warp reductions,
// the device status word and launch bookkeeping.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace gpt2 {

typedef __nv_bfloat16 bf16;

// Device status word bits (written by kernels with atomicOr, read by the host
// at the next synchronising call).
enum : unsigned {
    STATUS_BAD_TOKEN = 1u,
    STATUS_TIMEOUT = 2u,
};

// ---------------------------------------------------------------- conversions
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(bf16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }

// Load / store 4 consecutive elements (16 B for float, 8 B for bf16).
__device__ __forceinline__ void load4(const float* p, float v[4]) {
    float4 q = *reinterpret_cast<const float4*>(p);
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
}
__device__ __forceinline__ void load4(const bf16* p, float v[4]) {
    uint2 q = *reinterpret_cast<const uint2*>(p);
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&q.x);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&q.y);
    float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    v[0] = fa.x; v[1] = fa.y; v[2] = fb.x; v[3] = fb.y;
}
__device__ __forceinline__ void store4(float* p, const float v[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void store4(bf16* p, const float v[4]) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
    uint2 q;
    q.x = *reinterpret_cast<unsigned*>(&a);
    q.y = *reinterpret_cast<unsigned*>(&b);
    *reinterpret_cast<uint2*>(p) = q;
}

// Programmatic dependent launch (sm_90 and later). A kernel launched with the
// programmatic stream serialisation attribute may start while its predecessor
// in the stream still runs: griddep_wait blocks until that predecessor has
// completed and its writes are visible (a no-op for a kernel launched without
// the attribute), griddep_launch lets the next such kernel start. Every block
// of a kernel launched this way calls griddep_wait before it ends, so each
// kernel of a chain completes after all kernels before it.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------------ reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// GPT-2's tanh-approximated GELU and its derivative, evaluated in fp32 with
// CUDA's tanhf.
__device__ __forceinline__ float gelu_tanh(float u) {
    const float c = 0.7978845608028654f;  // sqrt(2/pi)
    float t = tanhf(c * (u + 0.044715f * u * u * u));
    return 0.5f * u * (1.0f + t);
}
__device__ __forceinline__ float gelu_tanh_grad(float u) {
    const float c = 0.7978845608028654f;
    float t = tanhf(c * (u + 0.044715f * u * u * u));
    return 0.5f * (1.0f + t) + 0.5f * u * (1.0f - t * t) * c * (1.0f + 3.0f * 0.044715f * u * u);
}

// The same GELU through the logistic identity 0.5 (1 + tanh z) = 1 / (1 + e^(-2z)):
// gelu(u) = u * s with s = sigmoid(2z), z = sqrt(2/pi) (u + 0.044715 u^3), and
// gelu'(u) = s + 2 u s (1 - s) sqrt(2/pi) (1 + 3 * 0.044715 u^2) since
// 1 - tanh(z)^2 = 4 s (1 - s). One exponential and one reciprocal, no
// cancellation in either tail. Used where the result is stored in bf16.
__device__ __forceinline__ float rcp_approx(float x) {   // hardware reciprocal (rcp.approx), 1/inf = 0
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ float gelu_sigmoid_s(float u) {
    const float c = 0.7978845608028654f;
    const float z = c * fmaf(0.044715f * u, u * u, u);
    return rcp_approx(1.0f + __expf(-2.0f * z));
}
__device__ __forceinline__ float gelu_fast(float u) { return u * gelu_sigmoid_s(u); }
__device__ __forceinline__ float gelu_fast_grad(float u) {
    const float c = 0.7978845608028654f;
    const float s = gelu_sigmoid_s(u);
    return fmaf(2.0f * u * s * (1.0f - s) * c, fmaf(3.0f * 0.044715f * u, u, 1.0f), s);
}
// GELU and its derivative from one exponential (logistic form).
__device__ __forceinline__ void gelu_fast_both(float u, float& g, float& dg) {
    const float c = 0.7978845608028654f;
    const float s = gelu_sigmoid_s(u);
    g = u * s;
    dg = fmaf(2.0f * u * s * (1.0f - s) * c, fmaf(3.0f * 0.044715f * u, u, 1.0f), s);
}
// Pairs of fp32 values in one 64-bit register, for the sm_100 packed fp32
// instructions (fma/mul/add .f32x2: one instruction per pair, IEEE
// round-to-nearest per lane like the scalar forms).
typedef unsigned long long f32x2;
__device__ __forceinline__ f32x2 pk2(float a, float b) {
    f32x2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void upk2(f32x2 v, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ f32x2 fma2(f32x2 a, f32x2 b, f32x2 c) {
    f32x2 r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b) {
    f32x2 r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ f32x2 add2(f32x2 a, f32x2 b) {
    f32x2 r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ float ex2_approx(float x) {   // hardware 2^x (ex2.approx), 2^-inf = 0
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// GELU (tanh form) and its derivative for two pre-activations, in the logistic
// form used by gelu_fast_both: s = 1 / (1 + 2^(u (K1 + K2 u^2))) with
// K1 = -2 c log2(e), K2 = 0.044715 K1 (so s = sigmoid(2 z), z = c (u + 0.044715 u^3));
// gelu = u s; gelu' = s + u s (1 - s) (2c + 6c 0.044715 u^2).
__device__ __forceinline__ void gelu_both_x2(float u0, float u1, float& g0, float& g1, float& d0, float& d1) {
    constexpr float c = 0.7978845608028654f;
    constexpr float K1 = -2.0f * c * 1.4426950408889634f;
    constexpr float K2 = K1 * 0.044715f;
    constexpr float K3 = 2.0f * c;
    constexpr float K4 = 6.0f * c * 0.044715f;
    const f32x2 U = pk2(u0, u1);
    const f32x2 U2 = mul2(U, U);
    const f32x2 Z = mul2(U, fma2(U2, pk2(K2, K2), pk2(K1, K1)));
    float z0, z1;
    upk2(Z, z0, z1);
    const f32x2 D = add2(pk2(ex2_approx(z0), ex2_approx(z1)), pk2(1.0f, 1.0f));
    float e0, e1;
    upk2(D, e0, e1);
    const f32x2 S = pk2(rcp_approx(e0), rcp_approx(e1));
    const f32x2 G = mul2(U, S);
    const f32x2 OMS = fma2(S, pk2(-1.0f, -1.0f), pk2(1.0f, 1.0f));
    const f32x2 Q = fma2(U2, pk2(K4, K4), pk2(K3, K3));
    const f32x2 DG = fma2(mul2(G, OMS), Q, S);
    upk2(G, g0, g1);
    upk2(DG, d0, d1);
}

// GELU and its derivative for an output element type: exact tanh form for fp32
// results, the logistic form for bf16 results.
template <typename T> __device__ __forceinline__ float gelu_for(float u);
template <> __device__ __forceinline__ float gelu_for<float>(float u) { return gelu_tanh(u); }
template <> __device__ __forceinline__ float gelu_for<bf16>(float u) { return gelu_fast(u); }
template <typename T> __device__ __forceinline__ float gelu_grad_for(float u);
template <> __device__ __forceinline__ float gelu_grad_for<float>(float u) { return gelu_tanh_grad(u); }
template <> __device__ __forceinline__ float gelu_grad_for<bf16>(float u) { return gelu_fast_grad(u); }

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ long long ceil_div_ll(long long a, long long b) { return (a + b - 1) / b; }

}  // namespace gpt2
