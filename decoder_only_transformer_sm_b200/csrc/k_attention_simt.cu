// SIMT causal attention, forward and backward, fp32 arithmetic: the fp32-mode
// attention (and the reference GPU path the tensor-core kernels are checked
// against). One thread owns one query row (forward, dQ) or one key row
// (dK, dV); K/V or Q/dO tiles are staged in shared memory. The softmax is
// computed online (running max and sum), so no T x T matrix is stored.
//
// Source definitions: "GPT-2 from Scratch", "CausalSelfAttention" (q, k, v are
// the three C-wide column blocks of the fused qkv projection; head h owns
// columns [h*hd, (h+1)*hd) of each block; att = softmax(q k^T / sqrt(hd)) with
// future positions masked to -inf; y = att v, heads concatenated back in head
// order) and "Let's reproduce GPT-2 (124M)", "FlashAttention and vocabulary
// padding" (online softmax, no materialised T x T matrix).
#include "kernels.cuh"

namespace gpt2 {

namespace {

constexpr int AT = 64;   // queries (or keys) per block = threads per block

template <typename T, int HD>
__global__ void __launch_bounds__(AT) attn_fwd_simt_kernel(const T* __restrict__ qkv, T* __restrict__ out,
                                                             float* __restrict__ lse, int Tn, int H) {
    __shared__ float Ks[AT][HD + 1];
    __shared__ float Vs[AT][HD + 1];
    const int bh = blockIdx.y, b = bh / H, h = bh % H;
    const int C = H * HD, ld = 3 * C;
    const int i = blockIdx.x * AT + threadIdx.x;
    const float scale = rsqrtf((float)HD);
    const T* base = qkv + (long long)b * Tn * ld;
    float q[HD], o[HD];
    float m = -INFINITY, l = 0.f;
#pragma unroll
    for (int d = 0; d < HD; ++d) {
        q[d] = (i < Tn) ? to_f(base[(long long)i * ld + h * HD + d]) * scale : 0.f;
        o[d] = 0.f;
    }
    const int jend = min(Tn, blockIdx.x * AT + AT);
    for (int j0 = 0; j0 < jend; j0 += AT) {
        const int j = j0 + threadIdx.x;
#pragma unroll
        for (int d = 0; d < HD; ++d) {
            Ks[threadIdx.x][d] = (j < Tn) ? to_f(base[(long long)j * ld + C + h * HD + d]) : 0.f;
            Vs[threadIdx.x][d] = (j < Tn) ? to_f(base[(long long)j * ld + 2 * C + h * HD + d]) : 0.f;
        }
        __syncthreads();
        if (i < Tn) {
            const int nj = min(AT, i - j0 + 1);
            for (int jj = 0; jj < nj; ++jj) {
                float s = 0.f;
#pragma unroll
                for (int d = 0; d < HD; ++d) s = fmaf(q[d], Ks[jj][d], s);
                const float mn = fmaxf(m, s);
                const float corr = expf(m - mn);
                const float p = expf(s - mn);
                l = l * corr + p;
#pragma unroll
                for (int d = 0; d < HD; ++d) o[d] = o[d] * corr + p * Vs[jj][d];
                m = mn;
            }
        }
        __syncthreads();
    }
    if (i < Tn) {
        const float inv = 1.f / l;
#pragma unroll
        for (int d = 0; d < HD; ++d) out[((long long)b * Tn + i) * C + h * HD + d] = from_f<T>(o[d] * inv);
        lse[(long long)bh * Tn + i] = m + logf(l);
    }
}

// D_i = sum_d dO_i,d * O_i,d   (per (b, h, i))
template <typename T, int HD>
__global__ void attn_bwd_pre_kernel(const T* __restrict__ out, const T* __restrict__ dout, float* __restrict__ dpre,
                                    int B, int Tn, int H) {
    const long long n = (long long)B * H * Tn;
    const long long g = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (g >= n) return;
    const int i = (int)(g % Tn);
    const int bh = (int)(g / Tn), b = bh / H, h = bh % H;
    const int C = H * HD;
    const long long r = ((long long)b * Tn + i) * C + h * HD;
    float s = 0.f;
#pragma unroll
    for (int d = 0; d < HD; ++d) s = fmaf(to_f(out[r + d]), to_f(dout[r + d]), s);
    dpre[g] = s;
}

// dQ_i = scale * sum_{j <= i} dS_ij k_j,  dS_ij = P_ij (dO_i . v_j - D_i),  P_ij = exp(S_ij - lse_i)
template <typename T, int HD>
__global__ void __launch_bounds__(AT) attn_bwd_dq_kernel(const T* __restrict__ qkv, const T* __restrict__ dout,
                                                           const float* __restrict__ lse,
                                                           const float* __restrict__ dpre, T* __restrict__ dqkv,
                                                           int Tn, int H) {
    __shared__ float Ks[AT][HD + 1];
    __shared__ float Vs[AT][HD + 1];
    const int bh = blockIdx.y, b = bh / H, h = bh % H;
    const int C = H * HD, ld = 3 * C;
    const int i = blockIdx.x * AT + threadIdx.x;
    const float scale = rsqrtf((float)HD);
    const T* base = qkv + (long long)b * Tn * ld;
    float q[HD], dO[HD], dq[HD];
    float L = 0.f, Dv = 0.f;
    if (i < Tn) { L = lse[(long long)bh * Tn + i]; Dv = dpre[(long long)bh * Tn + i]; }
#pragma unroll
    for (int d = 0; d < HD; ++d) {
        q[d] = (i < Tn) ? to_f(base[(long long)i * ld + h * HD + d]) * scale : 0.f;
        dO[d] = (i < Tn) ? to_f(dout[((long long)b * Tn + i) * C + h * HD + d]) : 0.f;
        dq[d] = 0.f;
    }
    const int jend = min(Tn, blockIdx.x * AT + AT);
    for (int j0 = 0; j0 < jend; j0 += AT) {
        const int j = j0 + threadIdx.x;
#pragma unroll
        for (int d = 0; d < HD; ++d) {
            Ks[threadIdx.x][d] = (j < Tn) ? to_f(base[(long long)j * ld + C + h * HD + d]) : 0.f;
            Vs[threadIdx.x][d] = (j < Tn) ? to_f(base[(long long)j * ld + 2 * C + h * HD + d]) : 0.f;
        }
        __syncthreads();
        if (i < Tn) {
            const int nj = min(AT, i - j0 + 1);
            for (int jj = 0; jj < nj; ++jj) {
                float s = 0.f, dp = 0.f;
#pragma unroll
                for (int d = 0; d < HD; ++d) { s = fmaf(q[d], Ks[jj][d], s); dp = fmaf(dO[d], Vs[jj][d], dp); }
                const float p = expf(s - L);
                const float ds = p * (dp - Dv);
#pragma unroll
                for (int d = 0; d < HD; ++d) dq[d] = fmaf(ds, Ks[jj][d], dq[d]);
            }
        }
        __syncthreads();
    }
    if (i < Tn) {
#pragma unroll
        for (int d = 0; d < HD; ++d) dqkv[((long long)b * Tn + i) * ld + h * HD + d] = from_f<T>(dq[d] * scale);
    }
}

// dV_j = sum_{i >= j} P_ij dO_i;  dK_j = scale * sum_{i >= j} dS_ij q_i
template <typename T, int HD>
__global__ void __launch_bounds__(AT) attn_bwd_dkv_kernel(const T* __restrict__ qkv, const T* __restrict__ dout,
                                                            const float* __restrict__ lse,
                                                            const float* __restrict__ dpre, T* __restrict__ dqkv,
                                                            int Tn, int H) {
    __shared__ float Qs[AT][HD + 1];
    __shared__ float Ds[AT][HD + 1];
    __shared__ float Ls[AT], Pd[AT];
    const int bh = blockIdx.y, b = bh / H, h = bh % H;
    const int C = H * HD, ld = 3 * C;
    const int j = blockIdx.x * AT + threadIdx.x;
    const float scale = rsqrtf((float)HD);
    const T* base = qkv + (long long)b * Tn * ld;
    float k[HD], v[HD], dk[HD], dv[HD];
#pragma unroll
    for (int d = 0; d < HD; ++d) {
        k[d] = (j < Tn) ? to_f(base[(long long)j * ld + C + h * HD + d]) : 0.f;
        v[d] = (j < Tn) ? to_f(base[(long long)j * ld + 2 * C + h * HD + d]) : 0.f;
        dk[d] = 0.f;
        dv[d] = 0.f;
    }
    const int istart = blockIdx.x * AT;
    for (int i0 = istart; i0 < Tn; i0 += AT) {
        const int i = i0 + threadIdx.x;
#pragma unroll
        for (int d = 0; d < HD; ++d) {
            Qs[threadIdx.x][d] = (i < Tn) ? to_f(base[(long long)i * ld + h * HD + d]) * scale : 0.f;
            Ds[threadIdx.x][d] = (i < Tn) ? to_f(dout[((long long)b * Tn + i) * C + h * HD + d]) : 0.f;
        }
        Ls[threadIdx.x] = (i < Tn) ? lse[(long long)bh * Tn + i] : 0.f;
        Pd[threadIdx.x] = (i < Tn) ? dpre[(long long)bh * Tn + i] : 0.f;
        __syncthreads();
        if (j < Tn) {
            const int ni = min(AT, Tn - i0);
            for (int ii = 0; ii < ni; ++ii) {
                if (i0 + ii < j) continue;
                float s = 0.f, dp = 0.f;
#pragma unroll
                for (int d = 0; d < HD; ++d) { s = fmaf(Qs[ii][d], k[d], s); dp = fmaf(Ds[ii][d], v[d], dp); }
                const float p = expf(s - Ls[ii]);
                const float ds = p * (dp - Pd[ii]);
#pragma unroll
                for (int d = 0; d < HD; ++d) {
                    dv[d] = fmaf(p, Ds[ii][d], dv[d]);
                    dk[d] = fmaf(ds, Qs[ii][d], dk[d]);   // Qs already carries the 1/sqrt(hd)
                }
            }
        }
        __syncthreads();
    }
    if (j < Tn) {
        const long long r = ((long long)b * Tn + j) * ld + h * HD;
#pragma unroll
        for (int d = 0; d < HD; ++d) {
            dqkv[r + C + d] = from_f<T>(dk[d]);
            dqkv[r + 2 * C + d] = from_f<T>(dv[d]);
        }
    }
}

}  // namespace

template <typename T>
void launch_attention_fwd_simt(const Ctx& ctx, const T* qkv, T* out, float* lse, int B, int Tn, int H, int hd) {
    dim3 grid(ceil_div(Tn, AT), B * H);
    if (hd == 64) attn_fwd_simt_kernel<T, 64><<<grid, AT, 0, ctx.stream>>>(qkv, out, lse, Tn, H);
    else attn_fwd_simt_kernel<T, 32><<<grid, AT, 0, ctx.stream>>>(qkv, out, lse, Tn, H);
    ++*ctx.launches;
}

template <typename T>
void launch_attention_bwd_simt(const Ctx& ctx, const T* qkv, const T* out, const T* dout, const float* lse,
                               float* dpre, T* dqkv, int B, int Tn, int H, int hd) {
    const long long n = (long long)B * H * Tn;
    dim3 grid(ceil_div(Tn, AT), B * H);
    if (hd == 64) {
        attn_bwd_pre_kernel<T, 64><<<(unsigned)ceil_div_ll(n, 256), 256, 0, ctx.stream>>>(out, dout, dpre, B, Tn, H);
        attn_bwd_dq_kernel<T, 64><<<grid, AT, 0, ctx.stream>>>(qkv, dout, lse, dpre, dqkv, Tn, H);
        attn_bwd_dkv_kernel<T, 64><<<grid, AT, 0, ctx.stream>>>(qkv, dout, lse, dpre, dqkv, Tn, H);
    } else {
        attn_bwd_pre_kernel<T, 32><<<(unsigned)ceil_div_ll(n, 256), 256, 0, ctx.stream>>>(out, dout, dpre, B, Tn, H);
        attn_bwd_dq_kernel<T, 32><<<grid, AT, 0, ctx.stream>>>(qkv, dout, lse, dpre, dqkv, Tn, H);
        attn_bwd_dkv_kernel<T, 32><<<grid, AT, 0, ctx.stream>>>(qkv, dout, lse, dpre, dqkv, Tn, H);
    }
    *ctx.launches += 3;
}

template void launch_attention_fwd_simt<float>(const Ctx&, const float*, float*, float*, int, int, int, int);
template void launch_attention_fwd_simt<bf16>(const Ctx&, const bf16*, bf16*, float*, int, int, int, int);
template void launch_attention_bwd_simt<float>(const Ctx&, const float*, const float*, const float*, const float*,
                                               float*, float*, int, int, int, int);
template void launch_attention_bwd_simt<bf16>(const Ctx&, const bf16*, const bf16*, const bf16*, const float*,
                                              float*, bf16*, int, int, int, int);

}  // namespace gpt2
