// One decode step of GPT-2 as one persistent kernel ("GPT-2 from Scratch",
// "A generation loop" on a key/value cache; the block of "The Block: pre-LN
// and residuals" with "CausalSelfAttention" and "The MLP and GPT-2's GELU";
// "Weight tying" for the logits). For B <= MEGA_MAX_B rows in bf16 with head
// width 64.
//
// Why one kernel: with one to four rows every GEMM of the step is a stream of
// its weights (250 MB at 124M) with a few multiply-adds per weight, and a step
// of separate kernels (five per layer) spends most of its time between them,
// each kernel's first loads waiting on the previous kernel's last stores.
// Here one CTA per SM runs the whole step; the five dependent phases of a
// layer are separated by grid barriers, and the weights do not wait for them:
// each CTA owns a fixed slice of rows of every weight matrix and a ring of
// MEGA_SLOTS shared-memory slots, and one thread keeps bulk copies
// (cp.async.bulk, completion on a slot's mbarrier) of its coming slices in
// flight, MEGA_SLOTS slices ahead, so the weight stream from HBM runs
// through the barriers.
//
// Phases of layer l (every CTA; "all rows" = the B rows of the step):
//   A  x = LN_1(resid) into shared memory (layer 0: resid = wte[tok] + wpe[pos]);
//      c_attn rows of this CTA: q, k, v of position pos into
//      the cache row (bias added, rounded to bf16).            -> grid barrier
//   B  attention of (b, h) = CTA index (B*H CTAs): q against cache rows
//      0 .. pos, online softmax over 64 key groups of 8 lanes, merged by
//      shuffles in each warp, then over the 16 warps -> att (bf16). -> grid barrier
//   C  att into shared memory; attn.c_proj rows: resid += att W^T + b.
//                                                               -> grid barrier
//   D  x = LN_2(resid); c_fc rows: fcg = gelu(bf16(x W^T + b)) (bf16).
//                                                               -> grid barrier
//   E  fcg into shared memory; mlp.c_proj rows: resid += fcg W^T + b.
//                                                               -> grid barrier
// then x = LN_f(resid) and the lm_head rows of this CTA (wte, tied), its
// slice streamed through the ring in chunks, into logits (bf16).
//
// Arithmetic per output is that of the other engines: fp32 dot products of
// bf16 operands, the epilogues of epilogue_scalar (bias then rounding; the
// residual add in fp32; GELU on the bf16-rounded pre-activation). Rows are
// reduced in a fixed order, so the step is deterministic.
//
// Grid barrier: one 64-bit count in global memory that only grows. Each launch
// passes 5 L barriers and each adds one per CTA, so between launches the count
// is a multiple of 5 L x grid; a CTA reads it at start (no CTA can pass the
// first barrier before every CTA has arrived, so the value read lies below
// the next multiple) and barrier i of the launch waits for base + (i+1) x grid.
// Arrival is a release add after the block barrier; the wait polls the count
// with acquire loads (bounded by wall time; on timeout the kernel sets
// STATUS_TIMEOUT and skips the remaining waits, and the host clears the count). Data written before a barrier by
// other CTAs is read after it through L2 (ld.global.cg). The launch is
// cooperative, so all CTAs are resident together.
//
// Latency: per phase, the loads that do not depend on the phase's input (the
// bias and residual elements of this CTA's rows, the layer table, read into
// shared memory once) are issued a job ahead, and a LayerNorm reads its row
// once into registers. Measured alternative, slower: each warp loading its
// next rows from HBM straight into registers (no ring) sped the lm_head up
// but slowed every other phase, the thousands of outstanding loads per SM
// queueing ahead of the phases' own loads.
#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace gpt2 {

namespace {

constexpr int MG_WARPS = 16;
constexpr int MG_THREADS = 32 * MG_WARPS;
constexpr int MG_HD = 64;
constexpr int MG_G = 8;                 // lanes per key in the attention (8 x 16 bytes = 64 bf16)
constexpr int MG_NG = MG_WARPS * 4;     // key groups per CTA
constexpr int MEGA_LN_NV = 8;           // float4 per lane of a LayerNorm row: C <= 1024

struct MegaSmem {
    unsigned char* ring;   // MEGA_SLOTS x MEGA_SLOT_BYTES
    bf16* xs;              // B x K operand rows (or the attention merge scratch)
    float* lnw;            // the next LayerNorm's weight (C floats) then bias (C floats)
    uint64_t* full;        // MEGA_SLOTS mbarriers
    int* issued;           // MEGA_SLOTS: the last job issued into each slot (-1: none)
    volatile uint32_t* abort;
    const DecodeLayer* layers;   // shared-memory copy of the layer table
    void* const* kv;             // shared-memory copy of the cache pointers
    unsigned long long* target;  // thread 0: the count the next barrier waits for
    int pos;               // the step's position
};

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     tc::smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void unpack8(const uint4& q, float* f) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 t = __bfloat1622float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

// Rows [row0, row0 + nrows) of a K-wide bf16 weight matrix: one ring job.
struct Job {
    const bf16* src;
    int row0, nrows, K, kind, layer;
};
enum { J_QKV = 0, J_PROJ = 1, J_FC = 2, J_FCP = 3, J_LM = 4 };

__device__ __forceinline__ Job job_of(const MegaDecode& p, const DecodeLayer* layers, int j) {
    Job jb;
    const int c = blockIdx.x, C = p.C;
    if (j < 4 * p.L) {
        const int l = j >> 2, kind = j & 3;
        const DecodeLayer& o = layers[l];
        const int N = kind == J_QKV ? 3 * C : kind == J_FC ? 4 * C : C;
        jb.K = kind == J_FCP ? 4 * C : C;
        const long long w = kind == J_QKV ? o.wqkv : kind == J_PROJ ? o.wproj : kind == J_FC ? o.wfc : o.wfcp;
        jb.row0 = min(N, c * p.rows[kind]);
        jb.nrows = min(N, jb.row0 + p.rows[kind]) - jb.row0;
        jb.src = p.W + w + (long long)jb.row0 * jb.K;
        jb.kind = kind;
        jb.layer = l;
    } else {
        const int i = j - 4 * p.L;
        const int base = min(p.V, c * p.rows_lm), end = min(p.V, base + p.rows_lm);
        jb.K = C;
        jb.row0 = min(end, base + i * p.chunk_lm);
        jb.nrows = min(end, jb.row0 + p.chunk_lm) - jb.row0;
        jb.src = p.W + p.off_wte + (long long)jb.row0 * C;
        jb.kind = J_LM;
        jb.layer = p.L;
    }
    return jb;
}

// One thread: start the copy of job j into slot j % MEGA_SLOTS.
__device__ __forceinline__ void issue(const MegaDecode& p, const MegaSmem& s, int j) {
    if (j >= 4 * p.L + p.n_lm) return;
    const Job jb = job_of(p, s.layers, j);
    const int slot = j % MEGA_SLOTS;
    const uint32_t bytes = (uint32_t)jb.nrows * jb.K * 2;
    s.issued[slot] = j;
    tc::mbar_expect_tx(&s.full[slot], bytes);
    unsigned char* dst = s.ring + (size_t)slot * MEGA_SLOT_BYTES;
    const unsigned char* src = reinterpret_cast<const unsigned char*>(jb.src);
    for (uint32_t off = 0; off < bytes; off += 16384u)
        bulk_g2s(dst + off, src + off, min(16384u, bytes - off), &s.full[slot]);
}

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* a) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(a) : "memory");
    return v;
}

__device__ void grid_sync(const MegaDecode& p, const MegaSmem& s) {
    __syncthreads();
    if (threadIdx.x == 0 && !*s.abort) {
        const unsigned long long target = *s.target + gridDim.x;
        *s.target = target;
        // release: this CTA's writes (ordered before thread 0 by the block barrier)
        // become visible before the arrival; the acquiring poll orders the reads after
        asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(p.bar) : "memory");
        if (ld_acquire_u64(p.bar) < target) {
            unsigned long long t0 = 0;
            for (uint32_t it = 0; ld_acquire_u64(p.bar) < target; ++it) {
                if ((it & 63u) == 63u) {
                    const unsigned long long now = tc::globaltimer();
                    if (t0 == 0) {
                        t0 = now;
                    } else if (now - t0 > tc::WAIT_LIMIT_NS) {
                        *s.abort = 1u;
                        atomicOr(p.status, STATUS_TIMEOUT);
                        break;
                    }
                }
            }
        }
    }
    __syncthreads();
}

// LayerNorm of the MB rows of resid (fp32, written by other CTAs) into xs, one
// warp per row (launch_layernorm_fwd's arithmetic and order), the row read
// once into registers.
template <int MB>
__device__ __forceinline__ void stage_ln(const MegaDecode& p, const MegaSmem& s, const float* src) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, C = p.C;
    asm volatile("cp.async.wait_all;" ::: "memory");   // this thread's part of the staged weights
    __syncthreads();                                     // everyone's
    const float* w = s.lnw;
    const float* b = s.lnw + C;
    if (warp < MB) {
        const float* x = src + (long long)warp * C;
        bf16* y = s.xs + (long long)warp * C;
        float4 v[MEGA_LN_NV];
#pragma unroll
        for (int i = 0; i < MEGA_LN_NV; ++i) {
            const int c = (lane + 32 * i) * 4;
            v[i] = c < C ? __ldcg(reinterpret_cast<const float4*>(x + c)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < MEGA_LN_NV; ++i) {
            sum += v[i].x;
            sum += v[i].y;
            sum += v[i].z;
            sum += v[i].w;
        }
        const float mu = warp_sum(sum) / C;
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < MEGA_LN_NV; ++i) {
            if ((lane + 32 * i) * 4 < C) {
                float d = v[i].x - mu;
                ss += d * d;
                d = v[i].y - mu;
                ss += d * d;
                d = v[i].z - mu;
                ss += d * d;
                d = v[i].w - mu;
                ss += d * d;
            }
        }
        const float rs = rsqrtf(warp_sum(ss) / C + 1e-5f);
#pragma unroll
        for (int i = 0; i < MEGA_LN_NV; ++i) {
            const int c = (lane + 32 * i) * 4;
            if (c < C) {
                float ww[4], bb[4], o[4];
                load4(w + c, ww);
                load4(b + c, bb);
                const float vv[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) o[j] = (vv[j] - mu) * rs * ww[j] + bb[j];
                store4(y + c, o);
            }
        }
    }
    __syncthreads();
}

// MB rows of K bf16 (written by other CTAs) into xs.
template <int MB>
__device__ __forceinline__ void stage_rows(const MegaSmem& s, const bf16* src, int K) {
    const int n16 = MB * K / 8;
    const uint4* in = reinterpret_cast<const uint4*>(src);
    uint4* out = reinterpret_cast<uint4*>(s.xs);
    for (int i = threadIdx.x; i < n16; i += MG_THREADS) out[i] = __ldcg(in + i);
    __syncthreads();
}

// Epilogue inputs of a job for this warp's first two rows r = warp + 16 i
// (i = 0, 1): lane 16 i + m (m < MB) holds the bias element and, for the
// residual GEMMs, resid[m, n]. Loaded one job ahead.
struct Pre {
    float b, r;
};

__device__ __forceinline__ long long bias_off(const DecodeLayer& o, int kind) {
    return kind == J_QKV ? o.bqkv : kind == J_PROJ ? o.bproj : kind == J_FC ? o.bfc : o.bfcp;
}

template <int MB>
__device__ __forceinline__ void preload(const MegaDecode& p, const MegaSmem& s, int j, Pre& pre) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (j >= 4 * p.L + p.n_lm) return;
    const Job jb = job_of(p, s.layers, j);
    if (jb.kind == J_LM) return;
    const int i = lane >> 4, m = lane & 15, r = warp + i * MG_WARPS;
    if (m < MB && r < jb.nrows) {
        const int n = jb.row0 + r;
        pre.b = p.P[bias_off(s.layers[jb.layer], jb.kind) + n];
        if (jb.kind == J_PROJ || jb.kind == J_FCP) pre.r = __ldcg(p.resid + (long long)m * p.C + n);
    }
}

// The weight and bias of the next LayerNorm into s.lnw a phase before it runs
// (cp.async, 16 bytes a thread; stage_ln waits for them). Its previous reader,
// the LayerNorm before, has finished: each LayerNorm ends with a block barrier.
__device__ __forceinline__ void stage_ln_weights(const MegaDecode& p, const MegaSmem& s, const float* w,
                                                 const float* b) {
    const int n16 = p.C / 4;
    for (int i = threadIdx.x; i < 2 * n16; i += MG_THREADS) {
        const float* src = i < n16 ? w + 4 * i : b + 4 * (i - n16);
        asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(tc::smem_u32(s.lnw + 4 * i)), "l"(src)
                     : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}

// Rows of job j from its ring slot against the MB operand rows in xs, then the
// job's epilogue; afterwards the slot takes job j + MEGA_SLOTS. A warp takes
// rows r and r + 16 in one pass (their loads, multiply-adds and shuffle
// reductions interleave); lanes 0..MB-1 finish row r and lanes 16..16+MB-1 row
// r + 16. The copy of the job that takes the freed slot is issued by thread 32
// (warp 1), off thread 0's path to the next grid barrier.
template <int MB>
__device__ __forceinline__ void gemv_job(const MegaDecode& p, const MegaSmem& s, int j, const Pre& pre) {
    const Job jb = job_of(p, s.layers, j);
    const int slot = j % MEGA_SLOTS;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int K = jb.K, K16 = K / 8, C = p.C;
    if (!*s.abort) tc::mbar_wait(&s.full[slot], (uint32_t)(j / MEGA_SLOTS) & 1u, s.abort, p.status);
    const uint4* wbase = reinterpret_cast<const uint4*>(s.ring + (size_t)slot * MEGA_SLOT_BYTES);
    const uint4* xr = reinterpret_cast<const uint4*>(s.xs);
    const long long boff = jb.kind == J_LM ? 0 : bias_off(s.layers[jb.layer], jb.kind);
    for (int r0 = warp; r0 < jb.nrows; r0 += 2 * MG_WARPS) {
        const int r1 = min(r0 + MG_WARPS, jb.nrows - 1);   // past the last row: a repeat, not stored
        const uint4* w0 = wbase + (long long)r0 * K16;
        const uint4* w1 = wbase + (long long)r1 * K16;
        float a0[MB], a1[MB];
#pragma unroll
        for (int m = 0; m < MB; ++m) a0[m] = a1[m] = 0.f;
#pragma unroll 4
        for (int q = lane; q < K16; q += 32) {
            float f0[8], f1[8];
            unpack8(w0[q], f0);
            unpack8(w1[q], f1);
#pragma unroll
            for (int m = 0; m < MB; ++m) {
                float x[8];
                unpack8(xr[m * K16 + q], x);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    a0[m] = fmaf(x[e], f0[e], a0[m]);
                    a1[m] = fmaf(x[e], f1[e], a1[m]);
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
            for (int m = 0; m < MB; ++m) {
                a0[m] += __shfl_xor_sync(0xffffffffu, a0[m], o);
                a1[m] += __shfl_xor_sync(0xffffffffu, a1[m], o);
            }
        }
        const int i = lane >> 4, m = lane & 15;
        const int r = i ? r0 + MG_WARPS : r0;
        if (m < MB && r < jb.nrows) {
            float a = i ? a1[0] : a0[0];
#pragma unroll
            for (int k = 1; k < MB; ++k)
                if (m == k) a = i ? a1[k] : a0[k];
            const int n = jb.row0 + r;
            const bool first = r0 == warp;   // the preloaded pass
            if (jb.kind == J_LM) {
                p.logits[(long long)m * p.V + n] = __float2bfloat16_rn(a);
            } else {
                const float bias = first ? pre.b : p.P[boff + n];
                if (jb.kind == J_QKV) {
                    bf16* row = static_cast<bf16*>(s.kv[jb.layer]) + ((long long)m * p.Tc + s.pos) * 3 * C;
                    row[n] = __float2bfloat16_rn(a + bias);
                } else if (jb.kind == J_FC) {
                    const float u = __bfloat162float(__float2bfloat16_rn(a + bias));
                    p.fcg[(long long)m * 4 * C + n] = __float2bfloat16_rn(gelu_for<bf16>(u));
                } else {
                    float* rs = p.resid + (long long)m * C + n;
                    const float old = first ? pre.r : __ldcg(rs);
                    *rs = old + (a + bias);
                }
            }
        }
    }
    __syncthreads();   // the slot and xs are free (the barrier orders the reads before the next copy)
    if (threadIdx.x == 32 && !*s.abort) issue(p, s, j + MEGA_SLOTS);
}

// Attention of the newest position of (b, h) = (blockIdx.x / H, blockIdx.x % H).
__device__ __forceinline__ void attention(const MegaDecode& p, const MegaSmem& s, int l) {
    const int bh = blockIdx.x;
    if (bh >= p.B * p.H) return;
    const int b = bh / p.H, h = bh % p.H, C = p.C;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int grp = warp * 4 + lane / MG_G, sub = lane % MG_G;
    const long long ld = 3LL * C;
    const bf16* seq = static_cast<const bf16*>(s.kv[l]) + (long long)b * p.Tc * ld;
    const int n = s.pos + 1;
    float* sm_m = reinterpret_cast<float*>(s.xs);
    float* sm_l = sm_m + MG_NG;
    float* sm_acc = sm_l + MG_NG;   // [MG_NG][MG_HD]
    float q[8];
    unpack8(__ldcg(reinterpret_cast<const uint4*>(seq + (long long)(n - 1) * ld + h * MG_HD + sub * 8)), q);
    const float sc = rsqrtf((float)MG_HD) * 1.4426950408889634f;   // scores in log2 units
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] *= sc;
    float m = -INFINITY, lsum = 0.f, acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    // the trip count is the same for the 8 lanes of a group (shuffles within it)
    for (int jb = 0; jb < n; jb += MG_NG * 2) {
        uint4 kq[2], vq[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int j = jb + u * MG_NG + grp;
            kq[u] = make_uint4(0, 0, 0, 0);
            vq[u] = make_uint4(0, 0, 0, 0);
            if (j < n) {
                const bf16* r = seq + (long long)j * ld + h * MG_HD + sub * 8;
                kq[u] = __ldcg(reinterpret_cast<const uint4*>(r + C));
                vq[u] = __ldcg(reinterpret_cast<const uint4*>(r + 2 * C));
            }
        }
        float scv[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            float k[8];
            unpack8(kq[u], k);
            float d = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) d = fmaf(q[i], k[i], d);
#pragma unroll
            for (int o = MG_G / 2; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
            scv[u] = (jb + u * MG_NG + grp < n) ? d : -INFINITY;
        }
        const float mx = fmaxf(m, fmaxf(scv[0], scv[1]));
        if (mx != -INFINITY) {
            const float corr = exp2f(m - mx);
            lsum *= corr;
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] *= corr;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const float pr = exp2f(scv[u] - mx);
                float v[8];
                unpack8(vq[u], v);
                lsum += pr;
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] = fmaf(pr, v[i], acc[i]);
            }
            m = mx;
        }
    }
    // merge the warp's four groups (lanes l, l + 8, l + 16, l + 24 hold the same dims)
#pragma unroll
    for (int o = MG_G; o < 32; o <<= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o), l2 = __shfl_xor_sync(0xffffffffu, lsum, o);
        const float M = fmaxf(m, m2);
        const float w1 = M == -INFINITY ? 0.f : exp2f(m - M), w2 = M == -INFINITY ? 0.f : exp2f(m2 - M);
        lsum = fmaf(lsum, w1, l2 * w2);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float a2 = __shfl_xor_sync(0xffffffffu, acc[i], o);
            acc[i] = fmaf(acc[i], w1, a2 * w2);
        }
        m = M;
    }
    if (lane < MG_G) {   // the warp's partial: (m, l, acc[64]) of its keys
        if (sub == 0) {
            sm_m[warp] = m;
            sm_l[warp] = lsum;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) sm_acc[warp * MG_HD + sub * 8 + i] = acc[i];
    }
    __syncthreads();
    if (threadIdx.x < MG_HD) {   // the 16 warp partials, in warp order
        const int d = threadIdx.x;
        float M = -INFINITY;
        for (int g = 0; g < MG_WARPS; ++g) M = fmaxf(M, sm_m[g]);   // finite: warp 0 holds key 0
        float L = 0.f, A = 0.f;
        for (int g = 0; g < MG_WARPS; ++g) {
            const float wgt = exp2f(sm_m[g] - M);
            L = fmaf(sm_l[g], wgt, L);
            A = fmaf(sm_acc[g * MG_HD + d], wgt, A);
        }
        p.att[(long long)b * C + h * MG_HD + d] = __float2bfloat16_rn(A / L);
    }
}

// The ops of one layer, in order; the step is L layers of them, then OP_LNF and
// n_lm lm_head jobs. Written as one loop over a switch so that each phase's
// code is in the kernel once (the instruction cache holds the whole loop).
enum {
    OP_LN1, OP_QKV, OP_SYNC1, OP_ATTN, OP_SYNC2, OP_STAGE_ATT, OP_PROJ, OP_SYNC3, OP_LN2, OP_FC, OP_SYNC4,
    OP_STAGE_FCG, OP_FCP, OP_SYNC5, OPS_PER_LAYER
};

template <int MB>
__global__ void __launch_bounds__(MG_THREADS, 1) decode_mega_kernel(const __grid_constant__ MegaDecode p) {
    extern __shared__ __align__(128) unsigned char mg_smem[];
    __shared__ uint32_t s_abort;
    __shared__ int s_issued[MEGA_SLOTS];
    __shared__ DecodeLayer s_layers[MEGA_MAX_L];
    __shared__ void* s_kv[MEGA_MAX_L];
    __shared__ unsigned long long s_target;
    MegaSmem s;
    s.ring = mg_smem;
    s.xs = reinterpret_cast<bf16*>(mg_smem + (size_t)MEGA_SLOTS * MEGA_SLOT_BYTES);
    s.full = reinterpret_cast<uint64_t*>(mg_smem + (size_t)MEGA_SLOTS * MEGA_SLOT_BYTES + MEGA_X_BYTES);
    s.lnw = reinterpret_cast<float*>(mg_smem + (size_t)MEGA_SLOTS * MEGA_SLOT_BYTES + MEGA_X_BYTES + 64);
    s.issued = s_issued;
    s.abort = &s_abort;
    s.layers = s_layers;
    s.kv = s_kv;
    s.target = &s_target;
    for (int i = threadIdx.x; i < p.L; i += MG_THREADS) {
        s_layers[i] = p.layers[i];
        s_kv[i] = p.kv[i];
    }
    __syncthreads();
    s.pos = p.pos_dev ? *p.pos_dev : p.pos_now;
    const int C = p.C, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        s_abort = 0;
        const unsigned long long per_launch = 5ull * p.L * gridDim.x, v = ld_acquire_u64(p.bar);
        s_target = v - v % per_launch;
        for (int i = 0; i < MEGA_SLOTS; ++i) {
            s_issued[i] = -1;
            tc::mbar_init(&s.full[i], 1);
        }
        tc::fence_barrier_init();
        // the weights do not depend on anything before this step: start at once
        for (int j = 0; j < MEGA_SLOTS; ++j) issue(p, s, j);
    }
    Pre cur = {0.f, 0.f}, nxt = cur;
    preload<MB>(p, s, 0, cur);
    __syncthreads();

    // layer 0's input: x = wte[tok] + wpe[pos], LN_1 of it into xs. Every CTA
    // also writes x as the residual stream (the same values), so the residual
    // elements this CTA preloads for attn.c_proj before the first barrier are
    // its own writes.
    if (warp < MB) {
        int tok = p.tok[warp];
        if (tok < 0 || tok >= p.V) {
            if (lane == 0) atomicOr(p.status, STATUS_BAD_TOKEN);
            tok = tok < 0 ? 0 : p.V - 1;
        }
        const float* te = p.P + p.off_wte + (long long)tok * C;
        const float* pe = p.P + p.off_wpe + (long long)s.pos * C;
        const float* w = p.P + s_layers[0].ln1w;
        const float* bb = p.P + s_layers[0].ln1b;
        float sum = 0.f;
        for (int c = lane * 4; c < C; c += 128) {
            float a[4], e[4];
            load4(te + c, a);
            load4(pe + c, e);
#pragma unroll
            for (int j = 0; j < 4; ++j) sum += a[j] + e[j];
        }
        const float mu = warp_sum(sum) / C;
        float ss = 0.f;
        for (int c = lane * 4; c < C; c += 128) {
            float a[4], e[4];
            load4(te + c, a);
            load4(pe + c, e);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float d = (a[j] + e[j]) - mu;
                ss += d * d;
            }
        }
        const float rs = rsqrtf(warp_sum(ss) / C + 1e-5f);
        for (int c = lane * 4; c < C; c += 128) {
            float a[4], e[4], ww[4], b4[4], x[4], o[4];
            load4(te + c, a);
            load4(pe + c, e);
            load4(w + c, ww);
            load4(bb + c, b4);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                x[j] = a[j] + e[j];
                o[j] = (x[j] - mu) * rs * ww[j] + b4[j];
            }
            store4(s.xs + (long long)warp * C + c, o);
            store4(p.resid + (long long)warp * C + c, x);
        }
    }
    __syncthreads();

    const int n_layer_ops = OPS_PER_LAYER * p.L;
    for (int t = 0; t < n_layer_ops + 1 + p.n_lm; ++t) {
        const int l = t < n_layer_ops ? t / OPS_PER_LAYER : p.L;
        const int op = t < n_layer_ops ? t % OPS_PER_LAYER : t == n_layer_ops ? -1 : -2;
        const DecodeLayer& o = s_layers[l < p.L ? l : 0];
        int job = -1;
        switch (op) {
        case OP_LN1:
            if (l > 0) stage_ln<MB>(p, s, p.resid);
            break;
        case OP_QKV:
            job = 4 * l + J_QKV;
            stage_ln_weights(p, s, p.P + o.ln2w, p.P + o.ln2b);
            break;
        case OP_ATTN:
            attention(p, s, l);
            break;
        case OP_STAGE_ATT:
            stage_rows<MB>(s, p.att, C);
            break;
        case OP_PROJ:
            job = 4 * l + J_PROJ;
            break;
        case OP_LN2:
            stage_ln<MB>(p, s, p.resid);
            break;
        case OP_FC:
            job = 4 * l + J_FC;
            if (l + 1 < p.L) stage_ln_weights(p, s, p.P + s_layers[l + 1].ln1w, p.P + s_layers[l + 1].ln1b);
            else stage_ln_weights(p, s, p.P + p.off_lnfw, p.P + p.off_lnfb);
            break;
        case OP_STAGE_FCG:
            stage_rows<MB>(s, p.fcg, 4 * C);
            break;
        case OP_FCP:
            job = 4 * l + J_FCP;
            break;
        case -1:
            stage_ln<MB>(p, s, p.resid);
            break;
        case -2:
            job = 4 * p.L + (t - n_layer_ops - 1);
            break;
        default:   // OP_SYNC1 .. OP_SYNC5
            grid_sync(p, s);
            break;
        }
        if (job >= 0) {
            preload<MB>(p, s, job + 1, nxt);
            gemv_job<MB>(p, s, job, cur);
            cur = nxt;
        }
    }
    // after a timeout, copies still in flight into this CTA's ring end before it
    // does (a fresh bounded wait per slot)
    if (threadIdx.x == 0 && *s.abort) {
        for (int i = 0; i < MEGA_SLOTS; ++i) {
            if (s_issued[i] < 0) continue;
            volatile uint32_t fresh = 0;
            tc::mbar_wait(&s.full[i], (uint32_t)(s_issued[i] / MEGA_SLOTS) & 1u, &fresh, p.status);
        }
    }
}

}  // namespace

// ring | operand rows | mbarriers (64 bytes) | LayerNorm weight and bias (C <= 1024)
size_t decode_mega_smem() { return (size_t)MEGA_SLOTS * MEGA_SLOT_BYTES + MEGA_X_BYTES + 64 + 2 * 1024 * 4; }

template <int MB>
static bool mega_fits_one() {
    int n = 0;
    const bool ok = cudaFuncSetAttribute(decode_mega_kernel<MB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)decode_mega_smem()) == cudaSuccess &&
                    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_mega_kernel<MB>, MG_THREADS,
                                                                  decode_mega_smem()) == cudaSuccess &&
                    n >= 1;
    cudaGetLastError();
    return ok;
}

// One CTA of each instantiation fits on an SM (shared memory set up once).
static bool mega_fits() {
    static int fits = -1;
    if (fits < 0) fits = mega_fits_one<1>() && mega_fits_one<2>() && mega_fits_one<3>() && mega_fits_one<4>();
    return fits == 1;
}

bool decode_mega_plan(MegaDecode& p, int num_sms) {
    if (p.B < 1 || p.B > MEGA_MAX_B || p.H < 1 || p.C % 8 != 0 || p.C != p.H * MG_HD) return false;
    if (p.L < 1 || p.L > MEGA_MAX_L || p.C > 128 * MEGA_LN_NV) return false;
    if (!mega_fits()) return false;
    const int G = num_sms;
    if (G < p.B * p.H) return false;
    const int C = p.C;
    const int N[4] = {3 * C, C, 4 * C, C};
    const int K[4] = {C, C, C, 4 * C};
    for (int k = 0; k < 4; ++k) {
        p.rows[k] = ceil_div(N[k], G);
        if ((long long)p.rows[k] * K[k] * 2 > MEGA_SLOT_BYTES) return false;
    }
    if ((long long)p.B * 4 * C * 2 > MEGA_X_BYTES) return false;
    if ((long long)(2 * MG_NG + MG_NG * MG_HD) * 4 > MEGA_X_BYTES) return false;
    p.rows_lm = ceil_div(p.V, G);
    p.chunk_lm = MEGA_SLOT_BYTES / (C * 2);
    p.n_lm = ceil_div(p.rows_lm, p.chunk_lm);
    p.grid = G;
    return true;
}

bool launch_decode_mega(const Ctx& ctx, const MegaDecode& p) {
    if (!mega_fits()) return false;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid);
    cfg.blockDim = dim3(MG_THREADS);
    cfg.dynamicSmemBytes = decode_mega_smem();
    cfg.stream = ctx.stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeCooperative;
    at[0].val.cooperative = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    cudaError_t e;
    switch (p.B) {
    case 1: e = cudaLaunchKernelEx(&cfg, decode_mega_kernel<1>, p); break;
    case 2: e = cudaLaunchKernelEx(&cfg, decode_mega_kernel<2>, p); break;
    case 3: e = cudaLaunchKernelEx(&cfg, decode_mega_kernel<3>, p); break;
    default: e = cudaLaunchKernelEx(&cfg, decode_mega_kernel<4>, p); break;
    }
    ++*ctx.launches;
    return e == cudaSuccess;
}

}  // namespace gpt2
