// Kernels of autoregressive generation ("GPT-2 from Scratch", "A generation
// loop"): attention of the newest position against a key/value cache, the
// sampling draw (temperature, top-k, one multinomial draw), and the row copies
// that fill the cache and move token windows.
//
// Cache layout: per layer (B, Tc, 3C) rows [q | k | v] in the activation type,
// row (b, j) at (b * Tc + j) * 3C, head h at columns h*hd of each C-wide block.
// Rows 0 .. n-1 of a sequence are its positions 0 .. n-1; the decode step's
// qkv GEMM writes row n-1 before the attention runs, and the attention reads q
// from that row and k, v from rows 0 .. n-1.
#include <climits>

#include <cooperative_groups.h>

#include "kernels.cuh"

namespace gpt2 {

namespace {

// 16 bytes of T unpacked to floats.
template <typename T> struct V16;
template <> struct V16<float> {
    static constexpr int N = 4;
    __device__ static void unpack(const uint4& q, float* f) {
        f[0] = __uint_as_float(q.x); f[1] = __uint_as_float(q.y);
        f[2] = __uint_as_float(q.z); f[3] = __uint_as_float(q.w);
    }
};
template <> struct V16<bf16> {
    static constexpr int N = 8;
    __device__ static void unpack(const uint4& q, float* f) {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 t = __bfloat1622float2(h[i]);
            f[2 * i] = t.x;
            f[2 * i + 1] = t.y;
        }
    }
};

constexpr int DEC_THREADS = 128;
constexpr int DEC_UNROLL = 4;

// Merge of the first Sn of the S partials of (b, h) = (bh / H, bh % H), head
// dim d: out = sum_s acc_s 2^(m_s - M) / sum_s l_s 2^(m_s - M), M = max_s m_s
// (finite: split 0 holds key 0). Reads through L2 (other blocks wrote part).
template <typename T, int HD>
__device__ __forceinline__ void combine_head(const float* part, int bh, int H, int C, int S, int Sn, int d,
                                             T* out) {
    const int b = bh / H, h = bh % H;
    const float* p = part + (long long)bh * S * (HD + 2);
    S = Sn;
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, __ldcg(p + s * (HD + 2)));
    float L = 0.f, A = 0.f;
    for (int s = 0; s < S; ++s) {
        const float w = exp2f(__ldcg(p + s * (HD + 2)) - M);
        L = fmaf(__ldcg(p + s * (HD + 2) + 1), w, L);
        A = fmaf(__ldcg(p + s * (HD + 2) + 2 + d), w, A);
    }
    out[(long long)b * C + h * HD + d] = from_f<T>(A / L);
}

// One block: keys [s*chunk, min(n, (s+1)*chunk)) of one (b, h). Groups of G
// lanes own one key at a time, each lane 16 bytes of its head dims; a group
// keeps an online softmax (running max m in log2 units, sum l, weighted sum of
// v); the block merges its groups and writes (m, l, acc[HD]) to part. With
// pos_dev the key count n is *pos_dev + 1, read here; a block whose range starts
// at or past n writes the empty partial (m = -inf, l = 0, acc = 0), which the
// combine weighs by zero. With counters, only the first S_act = ceil(n / chunk)
// blocks of (b, h) work (the others end at once); if S_act is 1 the block
// writes out itself, else the last of them to finish (a ticket taken after its
// partial is visible) merges the S_act partials into out and resets the counter.
template <typename T, int HD>
__global__ void __launch_bounds__(DEC_THREADS)
    attn_decode_partial_kernel(const T* __restrict__ cache, int H, int C, int Tc, int n, int chunk, int S,
                               float* __restrict__ part, const int* __restrict__ pos_dev, int* counters,
                               T* __restrict__ out) {
    constexpr int VE = V16<T>::N;
    constexpr int G = HD / VE;                       // lanes per key
    constexpr int KPW = 32 / G;                      // keys per warp per step
    constexpr int NG = (DEC_THREADS / 32) * KPW;     // key groups per block
    static_assert(G >= 1 && G <= 32 && 32 % G == 0, "head width and type give a bad lane split");
    __shared__ float sm_m[NG], sm_l[NG];
    __shared__ float sm_acc[NG][HD];

    const int bh = blockIdx.x, s = blockIdx.y;
    const int b = bh / H, h = bh % H;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gw = lane / G, sub = lane % G;
    const int grp = warp * KPW + gw;
    const long long ld = 3LL * C;
    const T* seq = cache + (long long)b * Tc * ld;
    __shared__ int s_last;
    griddep_launch();
    griddep_wait();
    if (pos_dev) n = *pos_dev + 1;
    const int S_act = counters ? (n + chunk - 1) / chunk : S;
    if (s >= S_act) return;

    float q[VE];
    {
        const uint4 qv = *reinterpret_cast<const uint4*>(seq + (long long)(n - 1) * ld + h * HD + sub * VE);
        V16<T>::unpack(qv, q);
        const float sc = rsqrtf((float)HD) * 1.4426950408889634f;   // scores in log2 units
#pragma unroll
        for (int i = 0; i < VE; ++i) q[i] *= sc;
    }
    const int j0 = s * chunk, j1 = min(n, j0 + chunk);
    float m = -INFINITY, l = 0.f, acc[VE];
#pragma unroll
    for (int i = 0; i < VE; ++i) acc[i] = 0.f;

    // the trip count is the same for every lane of the block (shuffles below)
    for (int jb = j0; jb < j1; jb += NG * DEC_UNROLL) {
        uint4 kq[DEC_UNROLL], vq[DEC_UNROLL];
#pragma unroll
        for (int u = 0; u < DEC_UNROLL; ++u) {
            const int j = jb + u * NG + grp;
            kq[u] = make_uint4(0, 0, 0, 0);
            vq[u] = make_uint4(0, 0, 0, 0);
            if (j < j1) {
                const T* r = seq + (long long)j * ld + h * HD + sub * VE;
                kq[u] = *reinterpret_cast<const uint4*>(r + C);
                vq[u] = *reinterpret_cast<const uint4*>(r + 2 * C);
            }
        }
        float sc[DEC_UNROLL];
#pragma unroll
        for (int u = 0; u < DEC_UNROLL; ++u) {
            float k[VE];
            V16<T>::unpack(kq[u], k);
            float d = 0.f;
#pragma unroll
            for (int i = 0; i < VE; ++i) d = fmaf(q[i], k[i], d);
#pragma unroll
            for (int o = G / 2; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
            sc[u] = (jb + u * NG + grp < j1) ? d : -INFINITY;
        }
        float mx = m;
#pragma unroll
        for (int u = 0; u < DEC_UNROLL; ++u) mx = fmaxf(mx, sc[u]);
        if (mx != -INFINITY) {   // same value on the G lanes of a group
            const float corr = exp2f(m - mx);
            l *= corr;
#pragma unroll
            for (int i = 0; i < VE; ++i) acc[i] *= corr;
#pragma unroll
            for (int u = 0; u < DEC_UNROLL; ++u) {
                const float p = exp2f(sc[u] - mx);
                float v[VE];
                V16<T>::unpack(vq[u], v);
                l += p;
#pragma unroll
                for (int i = 0; i < VE; ++i) acc[i] = fmaf(p, v[i], acc[i]);
            }
            m = mx;
        }
    }
    if (sub == 0) {
        sm_m[grp] = m;
        sm_l[grp] = l;
    }
#pragma unroll
    for (int i = 0; i < VE; ++i) sm_acc[grp][sub * VE + i] = acc[i];
    __syncthreads();
    if (threadIdx.x < HD) {
        const int d = threadIdx.x;
        float M = -INFINITY;
        for (int g = 0; g < NG; ++g) M = fmaxf(M, sm_m[g]);
        float L = 0.f, A = 0.f;
        if (M != -INFINITY) {   // else the block's key range is empty
            for (int g = 0; g < NG; ++g) {
                const float w = exp2f(sm_m[g] - M);
                L = fmaf(sm_l[g], w, L);
                A = fmaf(sm_acc[g][d], w, A);
            }
        }
        if (S_act == 1 && counters) {   // one split: its sums are the result (combine_head's arithmetic)
            out[(long long)b * C + h * HD + d] = from_f<T>(fmaf(A, 1.f, 0.f) / fmaf(L, 1.f, 0.f));
        } else {
            float* o = part + ((long long)bh * S + s) * (HD + 2);
            o[2 + d] = A;
            if (d == 0) {
                o[0] = M;
                o[1] = L;
            }
        }
    }
    if (!counters || S_act == 1) return;
    __threadfence();   // this block's partial, visible before its ticket
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&counters[bh], 1) == S_act - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (threadIdx.x < HD) combine_head<T, HD>(part, bh, H, C, S, S_act, threadIdx.x, out);
    if (threadIdx.x == 0) counters[bh] = 0;
}

// Merge the S partials of each (b, h): out = sum_s acc_s 2^(m_s - M) / sum_s l_s 2^(m_s - M).
template <typename T, int HD>
__global__ void attn_decode_combine_kernel(const float* __restrict__ part, int H, int C, int S, T* __restrict__ out) {
    griddep_launch();
    griddep_wait();
    combine_head<T, HD>(part, blockIdx.x, H, C, S, S, threadIdx.x, out);
}

// ------------------------------------------------------------------ sampling
constexpr int SMP_THREADS = 1024;

// Unsigned key with the order of the float values (-0 taken as +0).
__device__ __forceinline__ unsigned order_key(float f) {
    if (f == 0.f) f = 0.f;
    const unsigned u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The float a key stands for (order_key's inverse; -0 comes back as +0).
__device__ __forceinline__ float key_value(unsigned k) {
    return __uint_as_float((k & 0x80000000u) ? (k ^ 0x80000000u) : ~k);
}

// One block per row (rows too long for sample_cluster_kernel's shared memory).
// 1) top_k in [1, V): the key of the k-th largest value by a 4-pass radix
// select (8 bits a pass, high byte first; 2 passes for bf16); entries with a
// key at or above it are kept (ties at the k-th value stay). 2) The row maximum. 3) e_i =
// 2^((x_i - max) * log2(e) / temperature) over kept entries; thread t owns the
// contiguous indices [t*per, (t+1)*per); a block scan of the threads' sums
// gives each thread's starting cumulative value; the thread whose range holds
// u * total walks it in order to the first index whose cumulative value
// exceeds u * total. No thread claiming (rounding at the ends) gives the last
// kept index. With da, the uniform and the output slot are those of draw
// da->step of the call that da describes.
template <typename T>
__global__ void __launch_bounds__(SMP_THREADS)
    sample_kernel(const T* __restrict__ logits, long long ld, int V, float scale, int top_k,
                  const float* __restrict__ u, int* __restrict__ next, int* __restrict__ out, long long out_ld,
                  int out_col, const DecodeArgs* __restrict__ da) {
    __shared__ unsigned hist[256];
    __shared__ unsigned s_prefix, s_krem;
    __shared__ float s_wred[32];
    __shared__ int s_wredi[32];
    __shared__ float s_excl[SMP_THREADS + 1];
    __shared__ int s_pick;
    griddep_launch();
    griddep_wait();
    if (da) {
        u = da->u + (long long)da->step * gridDim.x;
        out = da->out;
        out_ld = da->out_ld;
        out_col = da->out_col0 + da->step;
    }
    const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const T* x = logits + (long long)row * ld;

    float mx;
    unsigned thr = 0;
    if (top_k >= 1 && top_k < V) {
        unsigned prefix = 0, mask = 0, krem = (unsigned)top_k;
        // bf16 values have keys whose low 16 bits are zero: two passes fix the key
        for (int shift = 24; shift >= (sizeof(T) == 2 ? 16 : 0); shift -= 8) {
            for (int i = tid; i < 256; i += SMP_THREADS) hist[i] = 0;
            __syncthreads();
            // Values of one row tend to share their high key bytes, so most keys of a
            // pass fall into a few bins: the lanes of a warp that hit one bin add once
            // (warp-aggregated), instead of 32 adds to one address.
            for (int i0 = 0; i0 < V; i0 += SMP_THREADS) {
                const int i = i0 + tid;
                unsigned bin = 256u;   // no bin: out of range, or outside the prefix
                if (i < V) {
                    const unsigned k = order_key(to_f(x[i]));
                    if ((k & mask) == prefix) bin = (k >> shift) & 255u;
                }
                const unsigned peers = __match_any_sync(0xffffffffu, bin);
                if (bin < 256u && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (unsigned)__popc(peers));
            }
            __syncthreads();
            // the digit: the largest d whose bins d..255 hold krem keys or more (0 if
            // none), krem minus the keys in the bins above it. Warp 0: lane l sums
            // bins 255 - 8l down to 248 - 8l; a scan over lanes finds the lane, which
            // walks its eight bins.
            if (warp == 0) {
                unsigned t = 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) t += hist[255 - 8 * lane - i];
                unsigned incl = t;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const unsigned n = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += n;
                }
                const unsigned hit = __ballot_sync(0xffffffffu, incl >= krem);
                const int L = hit ? __ffs(hit) - 1 : 31;
                if (lane == L) {
                    unsigned cum = incl - t;
                    int d = 255 - 8 * lane;
                    for (;; --d) {
                        if (d == 0 || cum + hist[d] >= krem) break;
                        cum += hist[d];
                    }
                    s_prefix = prefix | ((unsigned)d << shift);
                    s_krem = krem - cum;
                }
            }
            __syncthreads();
            prefix = s_prefix;
            krem = s_krem;
            mask |= 0xFFu << shift;
            __syncthreads();
        }
        thr = prefix;
    }

    {   // row maximum (always kept)
        mx = -INFINITY;
        for (int i = tid; i < V; i += SMP_THREADS) mx = fmaxf(mx, to_f(x[i]));
        mx = warp_max(mx);
        if (lane == 0) s_wred[warp] = mx;
        __syncthreads();
        if (warp == 0) {
            float v = s_wred[lane];
            v = warp_max(v);
            if (lane == 0) s_wred[0] = v;
        }
        __syncthreads();
        mx = s_wred[0];
        __syncthreads();
    }

    // per-thread sums over contiguous ranges
    const int per = (V + SMP_THREADS - 1) / SMP_THREADS;
    const int i0 = min(V, tid * per), i1 = min(V, i0 + per);
    float local = 0.f;
    int last_kept = -1;
    for (int i = i0; i < i1; ++i) {
        const float f = to_f(x[i]);
        if (order_key(f) >= thr) {
            local += exp2f((f - mx) * scale);
            last_kept = i;
        }
    }
    // exclusive scan of the thread sums
    float incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) s_wred[warp] = incl;
    int lk = last_kept;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lk = max(lk, __shfl_xor_sync(0xffffffffu, lk, o));
    if (lane == 0) s_wredi[warp] = lk;
    __syncthreads();
    if (warp == 0) {
        float w = s_wred[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float n = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += n;
        }
        s_wred[lane] = w;   // inclusive sums over warps
        int k = s_wredi[lane];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) k = max(k, __shfl_xor_sync(0xffffffffu, k, o));
        if (lane == 0) {
            s_wredi[0] = k;
            s_pick = INT_MAX;
        }
    }
    __syncthreads();
    const float woff = warp == 0 ? 0.f : s_wred[warp - 1];
    const float prev = __shfl_up_sync(0xffffffffu, incl, 1);
    s_excl[tid] = woff + (lane == 0 ? 0.f : prev);
    if (tid == SMP_THREADS - 1) s_excl[SMP_THREADS] = s_wred[31];
    __syncthreads();
    const float total = s_excl[SMP_THREADS];
    float uu = u[row];
    if (!(uu >= 0.f)) uu = 0.f;
    const float target = uu * total;
    const float lo = s_excl[tid], hi = s_excl[tid + 1];
    if (local > 0.f && lo <= target && target < hi) {
        float run = lo;
        int pick = last_kept;
        for (int i = i0; i < i1; ++i) {
            const float f = to_f(x[i]);
            if (order_key(f) >= thr) {
                run += exp2f((f - mx) * scale);
                if (run > target) {
                    pick = i;
                    break;
                }
            }
        }
        atomicMin(&s_pick, pick);
    }
    __syncthreads();
    if (tid == 0) {
        const int j = s_pick != INT_MAX ? s_pick : s_wredi[0];
        next[row] = j;
        if (out) out[(long long)row * out_ld + out_col] = j;
    }
}

// The same draw with one row split over a cluster of SMP_CS CTAs (blockIdx.x
// the rank, blockIdx.y the row): CTA r holds the order keys of its slice
// [r*slice, (r+1)*slice) in shared memory, and the CTAs exchange through
// distributed shared memory what the single-block kernel reduces over its
// threads: the slice maxima; per radix pass the slice histograms (each CTA's
// warp 0 adds the SMP_CS histograms and takes the digit, so every CTA holds
// the same prefix; the histograms alternate between two buffers, so a pass
// needs one cluster barrier); the slice sums, added in rank order, which give
// each slice its starting cumulative value and the total; and the slices'
// picks and last kept indices, which rank 0 reduces and writes. Thread t of a
// CTA owns a contiguous range of the slice as in the single-block kernel.
constexpr int SMP_CS = 8;
constexpr size_t SMP_STAGED_MAX = 216 * 1024;   // shared memory of a slice at most
inline int sample_slice(int V) { return ((V + SMP_CS - 1) / SMP_CS + 7) / 8 * 8; }

template <typename T>
__global__ void __launch_bounds__(SMP_THREADS)
    sample_cluster_kernel(const T* __restrict__ logits, long long ld, int V, int slice, float scale, int top_k,
                          const float* __restrict__ u, int* __restrict__ next, int* __restrict__ out,
                          long long out_ld, int out_col, const DecodeArgs* __restrict__ da) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    extern __shared__ unsigned s_keys[];   // this CTA's slice
    __shared__ unsigned hist[2][256];
    __shared__ unsigned s_kmax[32];
    __shared__ unsigned s_prefix, s_krem, s_cmax;
    __shared__ float s_wred[32];
    __shared__ int s_wredi[32];
    __shared__ float s_excl[SMP_THREADS + 1];
    __shared__ float s_total, s_off, s_gtot;
    __shared__ int s_last, s_glast, s_pick;
    griddep_launch();
    griddep_wait();
    const int rows = gridDim.y, row = blockIdx.y;
    const int rank = (int)cluster.block_rank();
    if (da) {
        u = da->u + (long long)da->step * rows;
        out = da->out;
        out_ld = da->out_ld;
        out_col = da->out_col0 + da->step;
    }
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const T* x = logits + (long long)row * ld;
    const int v0 = min(V, rank * slice), nloc = min(V, v0 + slice) - v0;

    // 0) the slice's keys and its largest key; the row maximum over the cluster
    unsigned kmax = 0;
    {
        constexpr int VE = 16 / sizeof(T);
        int done = 0;
        if ((reinterpret_cast<uintptr_t>(x + v0) & 15) == 0) {
            const int nv = nloc / VE;
            const uint4* xv = reinterpret_cast<const uint4*>(x + v0);
            for (int i = tid; i < nv; i += SMP_THREADS) {
                const uint4 q = xv[i];
                const T* e = reinterpret_cast<const T*>(&q);
#pragma unroll
                for (int j = 0; j < VE; ++j) {
                    const unsigned kk = order_key(to_f(e[j]));
                    s_keys[i * VE + j] = kk;
                    kmax = max(kmax, kk);
                }
            }
            done = nv * VE;
        }
        for (int i = done + tid; i < nloc; i += SMP_THREADS) {
            const unsigned kk = order_key(to_f(x[v0 + i]));
            s_keys[i] = kk;
            kmax = max(kmax, kk);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    if (lane == 0) s_kmax[warp] = kmax;
    __syncthreads();
    if (warp == 0) {
        unsigned k = s_kmax[lane];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) k = max(k, __shfl_xor_sync(0xffffffffu, k, o));
        if (lane == 0) s_cmax = k;
    }
    cluster.sync();
    unsigned gk = lane < SMP_CS ? *cluster.map_shared_rank(&s_cmax, lane) : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) gk = max(gk, __shfl_xor_sync(0xffffffffu, gk, o));
    const float mx = key_value(gk);   // the row maximum (always kept)

    // 1) the top-k threshold key
    unsigned thr = 0;
    if (top_k >= 1 && top_k < V) {
        unsigned prefix = 0, mask = 0, krem = (unsigned)top_k;
        int pass = 0;
        // bf16 values have keys whose low 16 bits are zero: two passes fix the key
        for (int shift = 24; shift >= (sizeof(T) == 2 ? 16 : 0); shift -= 8, ++pass) {
            unsigned* h = hist[pass & 1];
            for (int i = tid; i < 256; i += SMP_THREADS) h[i] = 0;
            __syncthreads();
            for (int i0 = 0; i0 < nloc; i0 += SMP_THREADS) {
                const int i = i0 + tid;
                unsigned bin = 256u;   // no bin: out of range, or outside the prefix
                if (i < nloc) {
                    const unsigned k = s_keys[i];
                    if ((k & mask) == prefix) bin = (k >> shift) & 255u;
                }
                const unsigned peers = __match_any_sync(0xffffffffu, bin);
                if (bin < 256u && lane == __ffs(peers) - 1) atomicAdd(&h[bin], (unsigned)__popc(peers));
            }
            cluster.sync();   // every slice's histogram of this pass is complete
            if (warp == 0) {
                unsigned hb[8], t = 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    hb[i] = 0;
                    for (int r = 0; r < SMP_CS; ++r) hb[i] += cluster.map_shared_rank(h, r)[255 - 8 * lane - i];
                    t += hb[i];
                }
                unsigned incl = t;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const unsigned n = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += n;
                }
                const unsigned hit = __ballot_sync(0xffffffffu, incl >= krem);
                const int L = hit ? __ffs(hit) - 1 : 31;
                if (lane == L) {
                    unsigned cum = incl - t;
                    int i = 0;
                    for (; i < 7; ++i) {
                        if (cum + hb[i] >= krem) break;
                        cum += hb[i];
                    }
                    s_prefix = prefix | ((unsigned)(255 - 8 * lane - i) << shift);
                    s_krem = krem - cum;
                }
            }
            __syncthreads();
            prefix = s_prefix;
            krem = s_krem;
            mask |= 0xFFu << shift;
        }
        thr = prefix;
    }

    // 2) sums over kept entries: per thread, per slice, then over the cluster
    const int per = (nloc + SMP_THREADS - 1) / SMP_THREADS;
    const int i0 = min(nloc, tid * per), i1 = min(nloc, i0 + per);
    float local = 0.f;
    int last_kept = -1;
    for (int i = i0; i < i1; ++i) {
        const unsigned k = s_keys[i];
        if (k >= thr) {
            local += exp2f((key_value(k) - mx) * scale);
            last_kept = v0 + i;
        }
    }
    float incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) s_wred[warp] = incl;
    int lk = last_kept;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lk = max(lk, __shfl_xor_sync(0xffffffffu, lk, o));
    if (lane == 0) s_wredi[warp] = lk;
    __syncthreads();
    if (warp == 0) {
        float w = s_wred[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float n = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += n;
        }
        s_wred[lane] = w;   // inclusive sums over warps
        int k = s_wredi[lane];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) k = max(k, __shfl_xor_sync(0xffffffffu, k, o));
        if (lane == 0) {
            s_last = k;
            s_pick = INT_MAX;
        }
        if (lane == 31) s_total = w;   // the slice's sum
    }
    __syncthreads();
    const float woff = warp == 0 ? 0.f : s_wred[warp - 1];
    const float prev = __shfl_up_sync(0xffffffffu, incl, 1);
    s_excl[tid] = woff + (lane == 0 ? 0.f : prev);
    if (tid == SMP_THREADS - 1) s_excl[SMP_THREADS] = s_wred[31];
    cluster.sync();   // slice sums and last kept indices visible to the cluster
    if (warp == 0) {   // lane r < SMP_CS reads slice r's; the sums are added in rank order
        const float t = lane < SMP_CS ? *cluster.map_shared_rank(&s_total, lane) : 0.f;
        int glk = lane < SMP_CS ? *cluster.map_shared_rank(&s_last, lane) : -1;
        float tot = 0.f, off = 0.f;
#pragma unroll
        for (int r = 0; r < SMP_CS; ++r) {
            if (r == rank) off = tot;
            tot += __shfl_sync(0xffffffffu, t, r);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) glk = max(glk, __shfl_xor_sync(0xffffffffu, glk, o));
        if (lane == 0) {
            s_off = off;
            s_gtot = tot;
            s_glast = glk;
        }
    }
    __syncthreads();

    // 3) the pick: the thread whose cumulative range holds u * total walks it
    const float off = s_off;
    float uu = u[row];
    if (!(uu >= 0.f)) uu = 0.f;
    const float target = uu * s_gtot;
    const float lo = off + s_excl[tid], hi = off + s_excl[tid + 1];
    if (local > 0.f && lo <= target && target < hi) {
        float run = lo;
        int pick = last_kept;
        for (int i = i0; i < i1; ++i) {
            const unsigned k = s_keys[i];
            if (k >= thr) {
                run += exp2f((key_value(k) - mx) * scale);
                if (run > target) {
                    pick = v0 + i;
                    break;
                }
            }
        }
        atomicMin(&s_pick, pick);
    }
    cluster.sync();   // every slice's pick
    if (rank == 0 && warp == 0) {
        int j = lane < SMP_CS ? *cluster.map_shared_rank(&s_pick, lane) : INT_MAX;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) j = min(j, __shfl_xor_sync(0xffffffffu, j, o));
        if (lane == 0) {
            if (j == INT_MAX) j = s_glast;
            next[row] = j;
            if (out) out[(long long)row * out_ld + out_col] = j;
        }
    }
    cluster.sync();   // rank 0's reads of the other slices are done before they exit
}

__global__ void decode_set_kernel(DecodeArgs* da, int pos, int step, const float* u, int* out, long long out_ld,
                                  int out_col0) {
    da->pos = pos;
    da->step = step;
    da->u = u;
    da->out = out;
    da->out_ld = out_ld;
    da->out_col0 = out_col0;
}

__global__ void decode_advance_kernel(DecodeArgs* da) {
    griddep_launch();
    griddep_wait();
    da->pos += 1;
    da->step += 1;
}

// ----------------------------------------------------------------- row copies
// k and v columns [C, 3C) of qkv row (b*Tn + t) of layer l -> cache row (b, t).
template <typename T>
__global__ void kv_store_kernel(const void* const* __restrict__ src, void* const* __restrict__ dst, int Tn, int Tc,
                                int C) {
    const int r = blockIdx.x, l = blockIdx.y;
    const int b = r / Tn, t = r % Tn;
    const long long ld = 3LL * C;
    const uint4* s = reinterpret_cast<const uint4*>(static_cast<const T*>(src[l]) + (long long)r * ld + C);
    uint4* d = reinterpret_cast<uint4*>(static_cast<T*>(dst[l]) + ((long long)b * Tc + t) * ld + C);
    const int n16 = (int)(2LL * C * sizeof(T) / 16);
    for (int i = threadIdx.x; i < n16; i += blockDim.x) d[i] = s[i];
}

__global__ void copy_tokens_kernel(const int* __restrict__ src, long long src_ld, int* __restrict__ dst,
                                   long long dst_ld, int cols) {
    const long long r = blockIdx.x;
    for (int c = threadIdx.x; c < cols; c += blockDim.x) dst[r * dst_ld + c] = src[r * src_ld + c];
}

}  // namespace

void attention_decode_split(int BH, int n, int num_sms, int* splits, int* chunk) {
    int want = ceil_div(2 * num_sms, BH);
    if (want < 1) want = 1;
    int s = min(want, ceil_div(n, DECODE_MIN_KEYS));
    if (s < 1) s = 1;
    const int c = ceil_div(n, s);
    *chunk = c;
    *splits = ceil_div(n, c);   // every split holds at least one key
}

template <typename T, int HD>
void launch_decode_hd(const Ctx& ctx, const T* cache, T* out, float* part, int B, int H, int Tc, int n, int chunk,
                      int S, const int* pos_dev, int* counters) {
    const int C = H * HD;
    launch_pdl(ctx, attn_decode_partial_kernel<T, HD>, dim3(B * H, S), dim3(DEC_THREADS), 0, cache, H, C, Tc, n,
               chunk, S, part, pos_dev, counters, out);
    ++*ctx.launches;
    if (!counters) {
        launch_pdl(ctx, attn_decode_combine_kernel<T, HD>, dim3(B * H), dim3(HD), 0, (const float*)part, H, C, S,
                   out);
        ++*ctx.launches;
    }
}

template <typename T>
void launch_attention_decode(const Ctx& ctx, const T* cache, T* out, float* part, int B, int H, int hd, int Tc,
                             int n, const int* pos_dev, int* counters) {
    if (pos_dev) n = Tc;   // split for the longest range; the kernel reads the true length
    int S = 1, chunk = n;
    attention_decode_split(B * H, n, ctx.num_sms, &S, &chunk);
    if (hd == 64) launch_decode_hd<T, 64>(ctx, cache, out, part, B, H, Tc, n, chunk, S, pos_dev, counters);
    else launch_decode_hd<T, 32>(ctx, cache, out, part, B, H, Tc, n, chunk, S, pos_dev, counters);
}

template <typename T>
void launch_sample(const Ctx& ctx, const T* logits, long long ld, int rows, int V, float temperature, int top_k,
                   const float* u, int* next, int* out, long long out_ld, int out_col, const DecodeArgs* da) {
    const float scale = 1.4426950408889634f / temperature;
    const int slice = sample_slice(V);
    const size_t smem = (size_t)slice * sizeof(unsigned);
    if (smem <= SMP_STAGED_MAX) {
        static bool attr = false;   // the attribute is per function; set once
        if (!attr) {
            cudaFuncSetAttribute(sample_cluster_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)SMP_STAGED_MAX);
            attr = true;
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(SMP_CS, rows);
        cfg.blockDim = dim3(SMP_THREADS);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = ctx.stream;
        cudaLaunchAttribute at[2];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = SMP_CS;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = at;
        cfg.numAttrs = ctx.pdl ? 2 : 1;
        cudaLaunchKernelEx(&cfg, sample_cluster_kernel<T>, logits, ld, V, slice, scale, top_k, u, next, out, out_ld,
                           out_col, da);
    } else {
        launch_pdl(ctx, sample_kernel<T>, dim3(rows), dim3(SMP_THREADS), 0, logits, ld, V, scale, top_k, u,
                   next, out, out_ld, out_col, da);
    }
    ++*ctx.launches;
}

void launch_decode_set(const Ctx& ctx, DecodeArgs* da, int pos, int step, const float* u, int* out,
                       long long out_ld, int out_col0) {
    decode_set_kernel<<<1, 1, 0, ctx.stream>>>(da, pos, step, u, out, out_ld, out_col0);
    ++*ctx.launches;
}

void launch_decode_advance(const Ctx& ctx, DecodeArgs* da) {
    launch_pdl(ctx, decode_advance_kernel, dim3(1), dim3(1), 0, da);
    ++*ctx.launches;
}

void launch_kv_store(const Ctx& ctx, const void* const* qkv_ptrs, void* const* cache_ptrs, int L, int B, int Tn,
                     int Tc, int C, int elem_size) {
    const dim3 grid(B * Tn, L);
    if (elem_size == 2)
        kv_store_kernel<bf16><<<grid, 128, 0, ctx.stream>>>(qkv_ptrs, cache_ptrs, Tn, Tc, C);
    else
        kv_store_kernel<float><<<grid, 128, 0, ctx.stream>>>(qkv_ptrs, cache_ptrs, Tn, Tc, C);
    ++*ctx.launches;
}

void launch_copy_tokens(const Ctx& ctx, const int* src, long long src_ld, int* dst, long long dst_ld, int rows,
                        int cols) {
    if (rows < 1 || cols < 1) return;
    copy_tokens_kernel<<<rows, 256, 0, ctx.stream>>>(src, src_ld, dst, dst_ld, cols);
    ++*ctx.launches;
}

#define INST(T)                                                                                                 \
    template void launch_attention_decode<T>(const Ctx&, const T*, T*, float*, int, int, int, int, int,         \
                                             const int*, int*);                                                 \
    template void launch_sample<T>(const Ctx&, const T*, long long, int, int, float, int, const float*, int*,   \
                                   int*, long long, int, const DecodeArgs*);
INST(float)
INST(bf16)
#undef INST

}  // namespace gpt2
