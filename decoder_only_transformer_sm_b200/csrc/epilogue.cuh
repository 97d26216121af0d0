// GEMM epilogue application, shared by the SIMT and the tensor-core GEMMs.
#pragma once

#include "kernels.cuh"

namespace gpt2 {

// Scalar epilogue for columns [col, col + n) of one row.
template <typename T>
__device__ __forceinline__ void epilogue_scalar(const Epilogue& ep, long long row, int col, int n,
                                                const float* acc) {
    const long long base = row * ep.ldo + col;
    for (int j = 0; j < n; ++j) {
        const float a = acc[j];
        switch (ep.kind) {
        case EPI_STORE: reinterpret_cast<T*>(ep.out)[base + j] = from_f<T>(a); break;
        case EPI_BIAS: reinterpret_cast<T*>(ep.out)[base + j] = from_f<T>(a + ep.bias[col + j]); break;
        case EPI_BIAS_GELU: {
            const float u = to_f(from_f<T>(a + ep.bias[col + j]));   // pre-activation as rounded
            reinterpret_cast<T*>(ep.out2)[base + j] = from_f<T>(gelu_grad_for<T>(u));
            reinterpret_cast<T*>(ep.out)[base + j] = from_f<T>(gelu_for<T>(u));
            break;
        }
        case EPI_BIAS_RESID:
            reinterpret_cast<float*>(ep.out)[base + j] = ep.resid[base + j] + (a + ep.bias[col + j]);
            break;
        case EPI_MUL:
            reinterpret_cast<T*>(ep.out)[base + j] = from_f<T>(a * to_f(reinterpret_cast<const T*>(ep.aux)[base + j]));
            break;
        case EPI_ACCUM_F32: {
            float* o = reinterpret_cast<float*>(ep.out) + base + j;
            if (ep.split_atomic) atomicAdd(o, a);
            else *o = (ep.beta != 0.f ? ep.beta * *o : 0.f) + a;
            break;
        }
        default: break;
        }
    }
}

// Four consecutive columns, all in range, 4-element aligned.
template <typename T>
__device__ __forceinline__ void epilogue_vec4(const Epilogue& ep, long long base, int col, const float* acc) {
    float v[4], b[4];
    switch (ep.kind) {
    case EPI_STORE:
        store4(reinterpret_cast<T*>(ep.out) + base, acc);
        break;
    case EPI_BIAS:
        load4(ep.bias + col, b);
        for (int j = 0; j < 4; ++j) v[j] = acc[j] + b[j];
        store4(reinterpret_cast<T*>(ep.out) + base, v);
        break;
    case EPI_BIAS_GELU: {
        float d[4];
        load4(ep.bias + col, b);
        for (int j = 0; j < 4; ++j) {
            const float u = to_f(from_f<T>(acc[j] + b[j]));   // pre-activation as rounded
            v[j] = gelu_for<T>(u);
            d[j] = gelu_grad_for<T>(u);
        }
        store4(reinterpret_cast<T*>(ep.out2) + base, d);
        store4(reinterpret_cast<T*>(ep.out) + base, v);
        break;
    }
    case EPI_BIAS_RESID: {
        float r[4];
        load4(ep.bias + col, b);
        load4(ep.resid + base, r);
        for (int j = 0; j < 4; ++j) v[j] = r[j] + (acc[j] + b[j]);
        store4(reinterpret_cast<float*>(ep.out) + base, v);
        break;
    }
    case EPI_MUL: {
        float u[4];
        load4(reinterpret_cast<const T*>(ep.aux) + base, u);
        for (int j = 0; j < 4; ++j) v[j] = acc[j] * u[j];
        store4(reinterpret_cast<T*>(ep.out) + base, v);
        break;
    }
    case EPI_ACCUM_F32: {
        float* o = reinterpret_cast<float*>(ep.out) + base;
        if (ep.split_atomic) {
            for (int j = 0; j < 4; ++j) atomicAdd(o + j, acc[j]);
            break;
        }
        if (ep.beta != 0.f) {
            float old[4];
            load4(o, old);
            for (int j = 0; j < 4; ++j) v[j] = ep.beta * old[j] + acc[j];
        } else {
            for (int j = 0; j < 4; ++j) v[j] = acc[j];
        }
        store4(o, v);
        break;
    }
    default: break;
    }
}

// Eight consecutive bf16 outputs as one 16-byte store.
__device__ __forceinline__ void store8(bf16* p, const float* v) {
    uint4 q;
    __nv_bfloat162 t[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) t[j] = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
    q.x = *reinterpret_cast<unsigned*>(&t[0]);
    q.y = *reinterpret_cast<unsigned*>(&t[1]);
    q.z = *reinterpret_cast<unsigned*>(&t[2]);
    q.w = *reinterpret_cast<unsigned*>(&t[3]);
    *reinterpret_cast<uint4*>(p) = q;
}
__device__ __forceinline__ void load8(const bf16* p, float* v) {
    const uint4 q = *reinterpret_cast<const uint4*>(p);
    const unsigned w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
        v[2 * j] = f.x;
        v[2 * j + 1] = f.y;
    }
}

// Eight consecutive columns with bf16 outputs (16-byte stores), in range and aligned.
__device__ __forceinline__ void epilogue_vec8_bf16(const Epilogue& ep, long long base, int col, const float* acc) {
    float v[8], b[8];
    switch (ep.kind) {
    case EPI_STORE:
        store8(reinterpret_cast<bf16*>(ep.out) + base, acc);
        break;
    case EPI_BIAS:
        load4(ep.bias + col, b);
        load4(ep.bias + col + 4, b + 4);
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = acc[j] + b[j];
        store8(reinterpret_cast<bf16*>(ep.out) + base, v);
        break;
    case EPI_BIAS_GELU: {
        float d[8];
        load4(ep.bias + col, b);
        load4(ep.bias + col + 4, b + 4);
#pragma unroll
        for (int j = 0; j < 8; ++j) gelu_fast_both(__bfloat162float(__float2bfloat16_rn(acc[j] + b[j])), v[j], d[j]);
        store8(reinterpret_cast<bf16*>(ep.out2) + base, d);
        store8(reinterpret_cast<bf16*>(ep.out) + base, v);
        break;
    }
    case EPI_MUL:
        load8(reinterpret_cast<const bf16*>(ep.aux) + base, b);
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = acc[j] * b[j];
        store8(reinterpret_cast<bf16*>(ep.out) + base, v);
        break;
    default:   // fp32 outputs
        epilogue_vec4<bf16>(ep, base, col, acc);
        epilogue_vec4<bf16>(ep, base + 4, col + 4, acc + 4);
        break;
    }
}

// Apply the epilogue to N_RUN consecutive columns [col, col + N_RUN) of one row.
// Columns at or beyond n_cols are skipped.
template <typename T, int N_RUN>
__device__ __forceinline__ void epilogue_run(const Epilogue& ep, long long row, int col, int n_cols,
                                             const float* acc) {
    const long long base = row * ep.ldo + col;
    if (sizeof(T) == 2 && N_RUN % 8 == 0 && col + N_RUN <= n_cols && (base & 7) == 0 && (col & 7) == 0) {
#pragma unroll
        for (int j = 0; j < N_RUN; j += 8) epilogue_vec8_bf16(ep, base + j, col + j, acc + j);
    } else if (col + N_RUN <= n_cols && (base & 3) == 0 && (col & 3) == 0) {
#pragma unroll
        for (int j = 0; j < N_RUN; j += 4) epilogue_vec4<T>(ep, base + j, col + j, acc + j);
    } else {
        epilogue_scalar<T>(ep, row, col, min(N_RUN, n_cols - col), acc);
    }
}

}  // namespace gpt2
