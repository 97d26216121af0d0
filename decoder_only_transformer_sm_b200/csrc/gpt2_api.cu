// Runtime and C ABI of the GPT-2 training step: owns every buffer of one model
// and enqueues the kernels of forward, loss, backward, clip and AdamW on the
// handle's stream.
//
// Step structure ("GPT-2 from Scratch": "The full model", "The Block: pre-LN and
// residuals", "The loop", "Gradient clipping", "AdamW, and weight decay on
// matrices only"; "Let's reproduce GPT-2 (124M)", "Gradient accumulation, and
// the bug in getting it right"):
//   x0 = wte[idx] + wpe[t]
//   per block: x += c_proj(attn(ln_1(x)));  x += mlp_c_proj(gelu(c_fc(ln_2(x))))
//   logits = ln_f(x) wte^T;  loss = mean CE over targets != -1
//   backward in reverse; grads accumulate (scaled by loss_scale per micro-batch)
//   norm = ||g||_2;  g *= min(1, clip / (norm + 1e-6));  AdamW.
#include "gpt2.h"
#include "kernels.cuh"

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <string>
#include <unordered_map>
#include <vector>

using namespace gpt2;

namespace {

thread_local std::string g_last_error;

int fail(int code, const std::string& msg) {
    g_last_error = msg;
    return code;
}

#define CK(call)                                                                                   \
    do {                                                                                           \
        cudaError_t e_ = (call);                                                                   \
        if (e_ != cudaSuccess) {                                                                   \
            return fail(GPT2_ERR_CUDA, std::string(#call) + ": " + cudaGetErrorString(e_));        \
        }                                                                                          \
    } while (0)

struct TensorRec {
    std::string name;
    int ndim;
    long long shape[2];
    long long offset;
    int decay;
};

struct DevScalars {
    double loss_accum;   // accumulated scaled training loss
    double fwd_loss;     // loss of the last forward-only call
    double sumsq;        // global gradient sum of squares
    int n_valid;         // targets != -1 in the current micro-batch
    unsigned status;     // STATUS_* bits
    int work;            // work-item counter of the attention backward
};

struct ProfSite {
    std::string name;
    long long launches = 0;
    double ms = 0, flops = 0, bytes = 0;
};

struct LayerOff {   // offsets of one block's tensors in the flat vector
    long long ln1w, ln1b, wqkv, bqkv, wproj, bproj, ln2w, ln2b, wfc, bfc, wfcp, bfcp;
};

}  // namespace

namespace gpt2 {
int set_error(int code, const char* msg) { return fail(code, msg); }
}  // namespace gpt2

struct gpt2_handle {
    gpt2_config cfg;
    cudaStream_t stream = nullptr;
    int device = 0, num_sms = 148;
    bool bf16_mode = false;
    int C = 0, L = 0, H = 0, hd = 0, V = 0, maxBT = 0;

    std::vector<TensorRec> tensors;
    std::vector<LayerOff> lo;
    long long off_wte = 0, off_wpe = 0, off_lnfw = 0, off_lnfb = 0;
    long long n_params = 0;

    float* params = nullptr;
    float* grads = nullptr;
    float* mom1 = nullptr;
    float* mom2 = nullptr;
    bf16* shadow = nullptr;
    AdamChunk* d_chunks = nullptr;
    int n_chunks = 0;

    // activations (element type = act type of the mode)
    char* act_pool = nullptr;
    std::vector<float*> resid;          // 2L+1 of (BT, C) fp32
    std::vector<float*> ln_mean, ln_rstd;  // 2L+1 of (BT)
    std::vector<void*> ln1, ln2, qkv, att, fch, fcg;  // per layer; fch = gelu'(u), fcg = gelu(u)
    std::vector<float*> lse;            // per layer (B, H, T)
    void* lnf = nullptr;
    void* logits = nullptr;
    float* dres = nullptr;
    void* dres_act = nullptr;
    void* dtmp = nullptr;
    void* dO = nullptr;
    void* dqkv = nullptr;
    void* du = nullptr;
    float* dpre = nullptr;
    float* red_scratch = nullptr;   // per-block partial column sums (LayerNorm bwd, bias grads)
    int* d_tokens = nullptr;

    DevScalars* d_sc = nullptr;
    DevScalars* h_sc = nullptr;   // pinned

    long long step_t = 0;
    long long launches = 0;
    bool use_tc_gemm = true;
    bool use_tc_attention = true;
    bool use_tcgen05_attention = true;        // tcgen05 forward for head width 64 (else the mma.sync kernel)
    bool use_tcgen05_attention_bwd = true;    // tcgen05 backward (faster than the mma.sync kernels)
    std::string host_error;   // set by enqueue helpers that cannot report a status

    // CUDA graph of zero_grad + forward + backward for one (B, T), captured on the
    // second step with that shape (the first runs eagerly, so one-time setup such
    // as kernel attributes happens outside a capture) and replayed afterwards.
    bool use_graphs = true;
    cudaStream_t cap_stream = nullptr;
    cudaGraphExec_t graph_exec = nullptr;
    int graph_B = 0, graph_T = 0;
    long long graph_launches = 0;

    // Generation ("A generation loop"): per layer a key/value cache of
    // (max_B, block_size, 3C) rows [q | k | v] in the activation type (the q
    // block of a row is written by the decode step's qkv GEMM and read only for
    // that row), allocated by the first prefill.
    char* gen_pool = nullptr;
    std::vector<void*> kv;
    void** d_layer_ptrs = nullptr;   // device [qkv[0..L-1], kv[0..L-1]] for the cache fill
    float* dec_part = nullptr;       // decode attention partial sums
    int* d_next = nullptr;           // last drawn token per row (max_B): the next decode step's input
    int* d_window = nullptr;         // contiguous token window of a prefill inside gpt2_generate (maxBT)
    int kv_B = 0, kv_len = 0;        // rows and positions the cache holds
    // gpt2_generate's decode steps read their position, draw index and output
    // slot from d_dec, so one captured step (decode, draw, advance of d_dec)
    // serves every position: captured on the second step with the same
    // (B, temperature, top_k) (the first runs the same launches eagerly).
    DecodeArgs* d_dec = nullptr;
    cudaGraphExec_t dec_graph = nullptr;
    bool dec_seen = false;
    int dec_B = 0, dec_top_k = 0;
    float dec_temperature = 0.f;
    long long dec_graph_launches = 0;
    int* dec_counters = nullptr;     // (max_B * H) tickets of the decode attention, zero between calls
    // bf16 decode steps of at most MEGA_MAX_B rows run as one persistent kernel
    // (decode_mega_kernel) when the shape fits; its layer offsets and barrier
    // words live in the generation pool
    bool use_mega = true;
    DecodeLayer* d_dec_layers = nullptr;
    unsigned long long* d_mega_bar = nullptr;
    bool pdl = false;                // launch_pdl kernels get programmatic dependent launch

    // Data-parallel exchange: caller-owned events recorded as each gradient bucket
    // becomes final in an eager backward (not inside a graph capture).
    std::vector<cudaEvent_t> grad_events;
    bool capturing = false;

    bool profiling = false;
    std::vector<ProfSite> psites;
    std::unordered_map<std::string, int> pidx;
    std::vector<cudaEvent_t> pev;
    size_t pev_used = 0;
    std::vector<std::pair<int, size_t>> ppending;

    Ctx ctx() {
        Ctx c;
        c.stream = stream;
        c.status = &d_sc->status;
        c.launches = &launches;
        c.num_sms = num_sms;
        c.pdl = pdl && !profiling;
        return c;
    }
};

// Programmatic dependent launch for the kernels enqueued while it lives (the
// generation path's chains of short kernels; see launch_pdl).
struct PdlScope {
    gpt2_handle* h;
    bool old;
    explicit PdlScope(gpt2_handle* hh) : h(hh), old(hh->pdl) { h->pdl = true; }
    ~PdlScope() { h->pdl = old; }
};

namespace {

// ---------------------------------------------------------------- validation
int validate_config(const gpt2_config* c) {
    if (!c) return fail(GPT2_ERR_INVALID_ARG, "cfg is NULL");
    if (c->n_layer < 1 || c->n_head < 1 || c->n_embd < 1 || c->vocab_size < 1 || c->block_size < 1 ||
        c->max_B < 1 || c->max_T < 1)
        return fail(GPT2_ERR_INVALID_ARG, "all sizes must be >= 1");
    if (c->n_embd % c->n_head != 0) return fail(GPT2_ERR_INVALID_ARG, "n_embd must be a multiple of n_head");
    const int hd = c->n_embd / c->n_head;
    if (hd != 32 && hd != 64) return fail(GPT2_ERR_INVALID_ARG, "head width n_embd/n_head must be 32 or 64");
    if (c->n_embd % 64 != 0) return fail(GPT2_ERR_INVALID_ARG, "n_embd must be a multiple of 64");
    if (c->n_embd > 2048) return fail(GPT2_ERR_INVALID_ARG, "n_embd must be <= 2048");
    if (c->vocab_size % 8 != 0) return fail(GPT2_ERR_INVALID_ARG, "vocab_size must be a multiple of 8 (pad it)");
    if (c->max_T > c->block_size) return fail(GPT2_ERR_INVALID_ARG, "max_T must be <= block_size");
    if (c->precision != GPT2_PRECISION_FP32 && c->precision != GPT2_PRECISION_BF16)
        return fail(GPT2_ERR_INVALID_ARG, "precision must be GPT2_PRECISION_FP32 or GPT2_PRECISION_BF16");
    if (c->flags != 0) return fail(GPT2_ERR_INVALID_ARG, "flags must be 0");
    if ((long long)c->max_B * c->max_T > (1LL << 30)) return fail(GPT2_ERR_INVALID_ARG, "max_B*max_T too large");
    return GPT2_OK;
}

int check_bt(const gpt2_handle* h, int B, int T) {
    if (B < 1 || T < 1) return fail(GPT2_ERR_INVALID_ARG, "B and T must be >= 1");
    if (B > h->cfg.max_B) return fail(GPT2_ERR_INVALID_ARG, "B exceeds max_B");
    if (T > h->cfg.max_T) return fail(GPT2_ERR_INVALID_ARG, "T exceeds max_T");
    if (T > h->cfg.block_size) return fail(GPT2_ERR_INVALID_ARG, "T exceeds block_size");
    if ((long long)B * T > h->maxBT) return fail(GPT2_ERR_INVALID_ARG, "B*T exceeds max_B*max_T");
    return GPT2_OK;
}

void build_layout(gpt2_handle* h) {
    const long long C = h->C, V = h->V;
    long long off = 0;
    auto add = [&](const std::string& name, long long r, long long c) {
        TensorRec t;
        t.name = name;
        t.ndim = c ? 2 : 1;
        t.shape[0] = r;
        t.shape[1] = c;
        t.offset = off;
        t.decay = c ? 1 : 0;
        h->tensors.push_back(t);
        long long o = off;
        off += c ? r * c : r;
        return o;
    };
    h->off_wte = add("wte", V, C);
    h->off_wpe = add("wpe", h->cfg.block_size, C);
    for (int l = 0; l < h->L; ++l) {
        std::string p = "h." + std::to_string(l) + ".";
        LayerOff o;
        o.ln1w = add(p + "ln_1.weight", C, 0);
        o.ln1b = add(p + "ln_1.bias", C, 0);
        o.wqkv = add(p + "attn.c_attn.weight", 3 * C, C);
        o.bqkv = add(p + "attn.c_attn.bias", 3 * C, 0);
        o.wproj = add(p + "attn.c_proj.weight", C, C);
        o.bproj = add(p + "attn.c_proj.bias", C, 0);
        o.ln2w = add(p + "ln_2.weight", C, 0);
        o.ln2b = add(p + "ln_2.bias", C, 0);
        o.wfc = add(p + "mlp.c_fc.weight", 4 * C, C);
        o.bfc = add(p + "mlp.c_fc.bias", 4 * C, 0);
        o.wfcp = add(p + "mlp.c_proj.weight", C, 4 * C);
        o.bfcp = add(p + "mlp.c_proj.bias", C, 0);
        h->lo.push_back(o);
    }
    h->off_lnfw = add("ln_f.weight", C, 0);
    h->off_lnfb = add("ln_f.bias", C, 0);
    h->n_params = off;
}

std::vector<AdamChunk> build_chunks(const gpt2_handle* h) {
    std::vector<AdamChunk> out;
    const long long CH = 1 << 16;
    for (const auto& t : h->tensors) {
        const long long n = t.ndim == 2 ? t.shape[0] * t.shape[1] : t.shape[0];
        for (long long s = 0; s < n; s += CH) {
            AdamChunk c;
            c.start = t.offset + s;
            c.count = (int)std::min(CH, n - s);
            c.decay = t.decay;
            out.push_back(c);
        }
    }
    return out;
}

size_t align_up(size_t x) { return (x + 255) & ~size_t(255); }

int init_weights(gpt2_handle* h) {
    Ctx c = h->ctx();
    const float resid_std = 0.02f / sqrtf(2.0f * h->L);
    for (size_t i = 0; i < h->tensors.size(); ++i) {
        const TensorRec& t = h->tensors[i];
        const long long n = t.ndim == 2 ? t.shape[0] * t.shape[1] : t.shape[0];
        float* p = h->params + t.offset;
        const bool is_ln = t.name.find("ln_") != std::string::npos;
        const bool is_weight = t.name.size() >= 6 && t.name.compare(t.name.size() - 6, 6, "weight") == 0;
        if (t.ndim == 2) {
            const bool resid_proj = t.name.size() >= 13 && t.name.compare(t.name.size() - 13, 13, "c_proj.weight") == 0;
            launch_fill_normal(c, p, n, resid_proj ? resid_std : 0.02f, h->cfg.seed, (unsigned long long)i);
        } else if (is_ln && is_weight) {
            launch_fill_const(c, p, n, 1.0f);
        } else {
            CK(cudaMemsetAsync(p, 0, n * sizeof(float), h->stream));
        }
    }
    CK(cudaGetLastError());
    return GPT2_OK;
}

int refresh_shadow(gpt2_handle* h) {
    if (!h->bf16_mode) return GPT2_OK;
    Ctx c = h->ctx();
    launch_to_bf16(c, h->params, h->shadow, h->n_params);
    CK(cudaGetLastError());
    return GPT2_OK;
}

// ----------------------------------------------------------- profiling
// With profiling on, every launch site is bracketed by two CUDA events on the
// handle's stream; the elapsed times are summed per site when the stream is
// next synchronised. flops/bytes are the algorithmic work of one launch.
int prof_site(gpt2_handle* h, const std::string& name) {
    auto it = h->pidx.find(name);
    if (it != h->pidx.end()) return it->second;
    ProfSite ps;
    ps.name = name;
    h->psites.push_back(ps);
    h->pidx[name] = (int)h->psites.size() - 1;
    return (int)h->psites.size() - 1;
}

template <class F>
void prof(gpt2_handle* h, const char* name, int M, int N, int K, double flops, double bytes, F&& launch) {
    if (!h->profiling || h->pev_used + 2 > h->pev.size()) {
        launch();
        return;
    }
    std::string nm(name);
    if (M > 0) nm += " " + std::to_string(M) + "x" + std::to_string(N) + "x" + std::to_string(K);
    const int site = prof_site(h, nm);
    ProfSite& ps = h->psites[site];
    ps.flops += flops;
    ps.bytes += bytes;
    ps.launches += 1;
    const size_t e = h->pev_used;
    cudaEventRecord(h->pev[e], h->stream);
    launch();
    cudaEventRecord(h->pev[e + 1], h->stream);
    h->pev_used += 2;
    h->ppending.push_back({site, e});
}

void prof_collect(gpt2_handle* h) {
    for (auto& pr : h->ppending) {
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, h->pev[pr.second], h->pev[pr.second + 1]) == cudaSuccess)
            h->psites[pr.first].ms += ms;
    }
    cudaGetLastError();
    h->ppending.clear();
    h->pev_used = 0;
}

#define PROF(name, M, N, K, flops, bytes, ...) prof(h, name, M, N, K, flops, bytes, [&]() { __VA_ARGS__; })

// ------------------------------------------------------------ GEMM dispatch
template <typename A>
void gemm_raw(gpt2_handle* h, GemmLayout layout, const void* a, const void* b, int M, int N, int K,
              const Epilogue& ep);

// A handful of rows (a decode step, last-position logits) on the weight-streaming
// kernel, which spreads the weight rows over every SM.
template <typename A>
bool gemm_few_rows(gpt2_handle* h, GemmLayout layout, const void* a, const void* b, int M, int N, int K,
                   const Epilogue& ep) {
    if (layout != GEMM_NT || !gemv_supported(sizeof(A), M, K) || ep.split_atomic) {
        if (ep.out_row_dev) {   // a device-picked output row needs this kernel
            h->host_error = "a GEMM with a device-side output row needs the weight-streaming kernel";
            return true;
        }
        return false;
    }
    launch_gemv<A>(h->ctx(), (const A*)a, (const A*)b, M, N, K, ep);
    return true;
}

template <>
void gemm_raw<float>(gpt2_handle* h, GemmLayout layout, const void* a, const void* b, int M, int N, int K,
                     const Epilogue& ep) {
    if (gemm_few_rows<float>(h, layout, a, b, M, N, K, ep)) return;
    launch_gemm_simt<float>(h->ctx(), layout, (const float*)a, (const float*)b, M, N, K, ep);
}

template <>
void gemm_raw<bf16>(gpt2_handle* h, GemmLayout layout, const void* a, const void* b, int M, int N, int K,
                    const Epilogue& ep) {
    if (gemm_few_rows<bf16>(h, layout, a, b, M, N, K, ep)) return;
    if (h->use_tc_gemm && gemm_tc_supported(layout, M, N, K)) {
        if (!launch_gemm_tc(h->ctx(), layout, (const bf16*)a, (const bf16*)b, M, N, K, ep))
            h->host_error = "tensor-map encoding failed for a tensor-core GEMM";
    } else {
        launch_gemm_simt<bf16>(h->ctx(), layout, (const bf16*)a, (const bf16*)b, M, N, K, ep);
    }
}

// Algorithmic bytes of one GEMM: operands once, the output once (read too for
// read-modify-write epilogues).
double gemm_bytes(int M, int N, int K, size_t es, const Epilogue& ep) {
    double b = ((double)M * K + (double)N * K) * es;
    const double mn = (double)M * N;
    switch (ep.kind) {
    case EPI_BIAS_GELU: b += 2 * mn * es; break;
    case EPI_BIAS_RESID: b += 2 * mn * 4; break;
    case EPI_MUL: b += 2 * mn * es; break;
    case EPI_ACCUM_F32: b += (ep.beta != 0.f ? 2 : 1) * mn * 4; break;
    default: b += mn * es; break;
    }
    return b;
}

// Whether gemm_raw<A> takes the tensor-core path for this shape.
template <typename A>
bool gemm_on_tc(gpt2_handle*, GemmLayout, int, int, int) {
    return false;
}
template <>
bool gemm_on_tc<bf16>(gpt2_handle* h, GemmLayout layout, int M, int N, int K) {
    return h->use_tc_gemm && gemm_tc_supported(layout, M, N, K);
}

template <typename A>
void gemm(gpt2_handle* h, const char* site, GemmLayout layout, const void* a, const void* b, int M, int N, int K,
          const Epilogue& ep) {
    PROF(site, M, N, K, 2.0 * M * N * K, gemm_bytes(M, N, K, sizeof(A), ep),
         gemm_raw<A>(h, layout, a, b, M, N, K, ep));
}

// Attention dispatch: tensor-core kernels in bf16 mode, SIMT fp32 kernels in fp32 mode.
template <typename A>
void attn_fwd(gpt2_handle* h, const A* qkv, A* out, float* lse, int B, int T);
template <>
void attn_fwd<float>(gpt2_handle* h, const float* qkv, float* out, float* lse, int B, int T) {
    launch_attention_fwd_simt<float>(h->ctx(), qkv, out, lse, B, T, h->H, h->hd);
}
template <>
void attn_fwd<bf16>(gpt2_handle* h, const bf16* qkv, bf16* out, float* lse, int B, int T) {
    if (!h->use_tc_attention) {
        launch_attention_fwd_simt<bf16>(h->ctx(), qkv, out, lse, B, T, h->H, h->hd);
    } else if (h->use_tcgen05_attention && attention_tc_supported(h->hd)) {
        if (!launch_attention_fwd_tc(h->ctx(), qkv, out, lse, B, T, h->H))
            h->host_error = "tensor-map encoding failed for the attention forward";
    } else {
        launch_attention_fwd_mma(h->ctx(), qkv, out, lse, B, T, h->H, h->hd);
    }
}
template <typename A>
void attn_bwd(gpt2_handle* h, const A* qkv, const A* out, const A* dout, const float* lse, A* dqkv, int B, int T,
              float* colsum_part);
// Whether attn_bwd<A> takes the tcgen05 path, which can also leave the column
// sums of dqkv (per 32-row group) in colsum_part.
template <typename A>
bool attn_bwd_sums(gpt2_handle*) {
    return false;
}
template <>
bool attn_bwd_sums<bf16>(gpt2_handle* h) {
    return h->use_tc_attention && h->use_tcgen05_attention_bwd && attention_tc_supported(h->hd);
}
template <>
void attn_bwd<float>(gpt2_handle* h, const float* qkv, const float* out, const float* dout, const float* lse,
                     float* dqkv, int B, int T, float*) {
    launch_attention_bwd_simt<float>(h->ctx(), qkv, out, dout, lse, h->dpre, dqkv, B, T, h->H, h->hd);
}
template <>
void attn_bwd<bf16>(gpt2_handle* h, const bf16* qkv, const bf16* out, const bf16* dout, const float* lse,
                    bf16* dqkv, int B, int T, float* colsum_part) {
    if (attn_bwd_sums<bf16>(h)) {
        // the fp32 dQ accumulator (B*T*C floats) lives in du, which is dead between the
        // c_fc input-gradient GEMM and the next block's mlp.c_proj backward
        if (!launch_attention_bwd_tc(h->ctx(), qkv, out, dout, lse, h->dpre, (float*)h->du, &h->d_sc->work, dqkv,
                                     B, T, h->H, colsum_part))
            h->host_error = "tensor-map encoding failed for the attention backward";
    } else if (h->use_tc_attention)
        launch_attention_bwd_mma(h->ctx(), qkv, out, dout, lse, h->dpre, dqkv, B, T, h->H, h->hd);
    else
        launch_attention_bwd_simt<bf16>(h->ctx(), qkv, out, dout, lse, h->dpre, dqkv, B, T, h->H, h->hd);
}

Epilogue epi(int kind, void* out, long long ldo) {
    Epilogue e;
    e.kind = kind;
    e.out = out;
    e.ldo = ldo;
    return e;
}

// Weight operand pointer: fp32 master (fp32 mode) or its bf16 copy (bf16 mode).
template <typename A> const A* wop(gpt2_handle* h, long long off);
template <> const float* wop<float>(gpt2_handle* h, long long off) { return h->params + off; }
template <> const bf16* wop<bf16>(gpt2_handle* h, long long off) { return h->shadow + off; }

// ------------------------------------------------------------------ forward
template <typename A>
void forward_impl(gpt2_handle* h, const int* idx, const int* targets, int B, int T, A* logits_out,
                  double* loss_slot, float loss_scale, bool write_grad, bool last_only = false) {
    Ctx c = h->ctx();
    const int BT = B * T, C = h->C, V = h->V, L = h->L, H = h->H, hd = h->hd;
    const double es = sizeof(A);
    const double ln_fwd_bytes = (double)BT * C * (4 + es) + 8.0 * BT;
    const double att_fwd_flops = 2.0 * B * H * (double)T * (T + 1) * hd;   // causal QK^T and PV
    float* P = h->params;
    PROF("embed+ln_1", 0, 0, 0, 0.0, (double)BT * C * (4 + 4 + 4 + es),
         launch_embed_ln<A>(c, idx, P + h->off_wte, P + h->off_wpe, BT, T, C, V, P + h->lo[0].ln1w,
                            P + h->lo[0].ln1b, h->resid[0], (A*)h->ln1[0], h->ln_mean[0], h->ln_rstd[0]));
    for (int l = 0; l < L; ++l) {
        const LayerOff& o = h->lo[l];
        Epilogue e = epi(EPI_BIAS, h->qkv[l], 3 * C);
        e.bias = P + o.bqkv;
        gemm<A>(h, "gemm fwd c_attn", GEMM_NT, h->ln1[l], wop<A>(h, o.wqkv), BT, 3 * C, C, e);
        PROF("attention fwd", 0, 0, 0, att_fwd_flops, (double)BT * C * es * 4,
             attn_fwd<A>(h, (const A*)h->qkv[l], (A*)h->att[l], h->lse[l], B, T));
        e = epi(EPI_BIAS_RESID, h->resid[2 * l + 1], C);
        e.bias = P + o.bproj;
        e.resid = h->resid[2 * l];
        gemm<A>(h, "gemm fwd attn.c_proj", GEMM_NT, h->att[l], wop<A>(h, o.wproj), BT, C, C, e);
        PROF("layernorm fwd", 0, 0, 0, 0.0, ln_fwd_bytes,
             launch_layernorm_fwd<A>(c, h->resid[2 * l + 1], P + o.ln2w, P + o.ln2b, (A*)h->ln2[l],
                                     h->ln_mean[2 * l + 1], h->ln_rstd[2 * l + 1], BT, C));
        e = epi(EPI_BIAS_GELU, h->fcg[l], 4 * C);
        e.out2 = h->fch[l];
        e.bias = P + o.bfc;
        gemm<A>(h, "gemm fwd c_fc+gelu", GEMM_NT, h->ln2[l], wop<A>(h, o.wfc), BT, 4 * C, C, e);
        e = epi(EPI_BIAS_RESID, h->resid[2 * l + 2], C);
        e.bias = P + o.bfcp;
        e.resid = h->resid[2 * l + 1];
        gemm<A>(h, "gemm fwd mlp.c_proj", GEMM_NT, h->fcg[l], wop<A>(h, o.wfcp), BT, C, 4 * C, e);
        const bool last = (l + 1 == L);
        PROF("layernorm fwd", 0, 0, 0, 0.0, ln_fwd_bytes,
             launch_layernorm_fwd<A>(c, h->resid[2 * l + 2], last ? P + h->off_lnfw : P + h->lo[l + 1].ln1w,
                                     last ? P + h->off_lnfb : P + h->lo[l + 1].ln1b,
                                     last ? (A*)h->lnf : (A*)h->ln1[l + 1], h->ln_mean[2 * l + 2],
                                     h->ln_rstd[2 * l + 2], BT, C));
    }
    if (last_only) {   // logits of each sequence's last position only: (B, V)
        PROF("gather last rows", 0, 0, 0, 0.0, 2.0 * B * C * es,
             launch_gather_last_rows<A>(c, (const A*)h->lnf, B, T, C, (A*)h->dtmp));
        gemm<A>(h, "gemm fwd lm_head (last position)", GEMM_NT, h->dtmp, wop<A>(h, h->off_wte), B, V, C,
                epi(EPI_STORE, logits_out, V));
        return;
    }
    A* lg = logits_out ? logits_out : (A*)h->logits;
    gemm<A>(h, "gemm fwd lm_head", GEMM_NT, h->lnf, wop<A>(h, h->off_wte), BT, V, C, epi(EPI_STORE, lg, V));
    if (targets) {
        PROF("count targets", 0, 0, 0, 0.0, 4.0 * BT, launch_count_targets(c, targets, BT, V, &h->d_sc->n_valid));
        PROF("classifier", 0, 0, 0, 0.0, (double)BT * V * es * (write_grad ? 2 : 1),
             launch_classifier<A>(c, lg, targets, BT, V, &h->d_sc->n_valid, loss_scale, loss_slot,
                                  write_grad ? 1 : 0));
    }
}

// ----------------------------------------------------------------- backward
// Gradient buckets in the order the backward finishes them: ln_f, block L-1, ...,
// block 0, then wte and wpe (the embedding backward adds into the tied wte last).
void grad_buckets(const gpt2_handle* h, std::vector<std::pair<long long, long long>>& out) {
    out.clear();
    out.push_back({h->off_lnfw, h->n_params - h->off_lnfw});
    for (int l = h->L - 1; l >= 0; --l) {
        const long long end = l + 1 < h->L ? h->lo[l + 1].ln1w : h->off_lnfw;
        out.push_back({h->lo[l].ln1w, end - h->lo[l].ln1w});
    }
    out.push_back({0, h->lo[0].ln1w});
}

// Bucket k of grad_buckets is final: record the caller's event k.
void bucket_done(gpt2_handle* h, int k) {
    if (!h->grad_events.empty() && !h->capturing) cudaEventRecord(h->grad_events[k], h->stream);
}

template <typename A>
void backward_impl(gpt2_handle* h, const int* idx, int B, int T) {
    Ctx c = h->ctx();
    const int BT = B * T, C = h->C, V = h->V, L = h->L, H = h->H, hd = h->hd;
    const double es = sizeof(A);
    const double ln_bwd_bytes = (double)BT * C * (es + 4 + 4 + 4 + es);
    const double att_bwd_flops = 5.0 * B * H * (double)T * (T + 1) * hd;   // S recompute, dV, dP, dQ, dK
    float* P = h->params;
    float* G = h->grads;
    // lm_head (tied): dlnf = dlogits wte ; dwte += dlogits^T lnf
    gemm<A>(h, "gemm dgrad lm_head", GEMM_NN, h->logits, wop<A>(h, h->off_wte), BT, C, V,
            epi(EPI_STORE, h->dtmp, C));
    Epilogue acc = epi(EPI_ACCUM_F32, G + h->off_wte, C);
    acc.beta = 1.f;
    gemm<A>(h, "gemm wgrad lm_head", GEMM_TN, h->logits, h->lnf, V, C, BT, acc);
    PROF("layernorm bwd", 0, 0, 0, 0.0, ln_bwd_bytes - 4.0 * BT * C,
         launch_layernorm_bwd<A>(c, (const A*)h->dtmp, h->resid[2 * L], h->ln_mean[2 * L], h->ln_rstd[2 * L],
                                 P + h->off_lnfw, nullptr, h->dres, (A*)h->dres_act, G + h->off_lnfw,
                                 G + h->off_lnfb, G + h->lo[L - 1].bfcp, BT, C, h->red_scratch));
    bucket_done(h, 0);   // ln_f
    for (int l = L - 1; l >= 0; --l) {
        const LayerOff& o = h->lo[l];
        // mlp.c_proj: dW += dY^T g ; du = (dY W) * gelu'(u)
        acc = epi(EPI_ACCUM_F32, G + o.wfcp, 4 * C);
        acc.beta = 1.f;
        gemm<A>(h, "gemm wgrad mlp.c_proj", GEMM_TN, h->dres_act, h->fcg[l], C, 4 * C, BT, acc);
        Epilogue e = epi(EPI_MUL, h->du, 4 * C);   // du = (dY W) * gelu'(u), gelu'(u) stored by the forward
        e.aux = h->fch[l];
        // on the tensor-core path the epilogue also leaves per-32-row column sums of du
        // (the c_fc bias gradient) in red_scratch
        const bool fused_colsum = gemm_on_tc<A>(h, GEMM_NN, BT, 4 * C, C);
        if (fused_colsum) e.colsum_part = h->red_scratch;
        gemm<A>(h, "gemm dgrad mlp.c_proj*gelu'", GEMM_NN, h->dres_act, wop<A>(h, o.wfcp), BT, 4 * C, C, e);
        if (fused_colsum) {
            PROF("bias colsum", 0, 0, 0, 0.0, (double)ceil_div(BT, 32) * 4 * C * 4,
                 launch_colred_finalize(c, h->red_scratch, ceil_div(BT, 32), 4 * C, G + o.bfc));
        } else {
            PROF("bias colsum", 0, 0, 0, 0.0, (double)BT * 4 * C * es,
                 launch_colsum<A>(c, (const A*)h->du, BT, 4 * C, G + o.bfc, h->red_scratch));
        }
        // mlp.c_fc: dW += du^T ln2 ; dln2 = du W
        acc = epi(EPI_ACCUM_F32, G + o.wfc, C);
        acc.beta = 1.f;
        gemm<A>(h, "gemm wgrad c_fc", GEMM_TN, h->du, h->ln2[l], 4 * C, C, BT, acc);
        gemm<A>(h, "gemm dgrad c_fc", GEMM_NN, h->du, wop<A>(h, o.wfc), BT, C, 4 * C, epi(EPI_STORE, h->dtmp, C));
        // ln_2 backward + residual; colsum of the result is the attn.c_proj bias gradient
        PROF("layernorm bwd", 0, 0, 0, 0.0, ln_bwd_bytes,
             launch_layernorm_bwd<A>(c, (const A*)h->dtmp, h->resid[2 * l + 1], h->ln_mean[2 * l + 1],
                                     h->ln_rstd[2 * l + 1], P + o.ln2w, h->dres, h->dres, (A*)h->dres_act,
                                     G + o.ln2w, G + o.ln2b, G + o.bproj, BT, C, h->red_scratch));
        // attn.c_proj
        acc = epi(EPI_ACCUM_F32, G + o.wproj, C);
        acc.beta = 1.f;
        gemm<A>(h, "gemm wgrad attn.c_proj", GEMM_TN, h->dres_act, h->att[l], C, C, BT, acc);
        gemm<A>(h, "gemm dgrad attn.c_proj", GEMM_NN, h->dres_act, wop<A>(h, o.wproj), BT, C, C,
                epi(EPI_STORE, h->dO, C));
        // attention
        // on the tcgen05 path the backward also leaves per-32-row column sums of dqkv
        // (the c_attn bias gradient) in red_scratch
        const bool attn_sums = attn_bwd_sums<A>(h);
        PROF("attention bwd", 0, 0, 0, att_bwd_flops, (double)BT * C * es * 8,
             attn_bwd<A>(h, (const A*)h->qkv[l], (const A*)h->att[l], (const A*)h->dO, h->lse[l], (A*)h->dqkv, B,
                         T, attn_sums ? h->red_scratch : nullptr));
        if (attn_sums) {
            const int groups = B * ceil_div(T, 32);
            PROF("bias colsum", 0, 0, 0, 0.0, (double)groups * 3 * C * 4,
                 launch_colred_finalize(c, h->red_scratch, groups, 3 * C, G + o.bqkv));
        } else {
            PROF("bias colsum", 0, 0, 0, 0.0, (double)BT * 3 * C * es,
                 launch_colsum<A>(c, (const A*)h->dqkv, BT, 3 * C, G + o.bqkv, h->red_scratch));
        }
        // attn.c_attn
        acc = epi(EPI_ACCUM_F32, G + o.wqkv, C);
        acc.beta = 1.f;
        gemm<A>(h, "gemm wgrad c_attn", GEMM_TN, h->dqkv, h->ln1[l], 3 * C, C, BT, acc);
        gemm<A>(h, "gemm dgrad c_attn", GEMM_NN, h->dqkv, wop<A>(h, o.wqkv), BT, C, 3 * C,
                epi(EPI_STORE, h->dtmp, C));
        // ln_1 backward + residual; colsum is the previous block's mlp.c_proj bias gradient
        PROF("layernorm bwd", 0, 0, 0, 0.0, ln_bwd_bytes,
             launch_layernorm_bwd<A>(c, (const A*)h->dtmp, h->resid[2 * l], h->ln_mean[2 * l], h->ln_rstd[2 * l],
                                     P + o.ln1w, h->dres, h->dres, (A*)h->dres_act, G + o.ln1w, G + o.ln1b,
                                     l > 0 ? G + h->lo[l - 1].bfcp : nullptr, BT, C, h->red_scratch));
        bucket_done(h, L - l);   // block l (its mlp.c_proj bias gradient was added by block l+1 or ln_f)
    }
    // deterministic: the GELU-backward buffer (free by now; BT x 4C elements of at least
    // 2 bytes, so at least BT x 8C bytes) holds the per-run partial sums and the sort.
    // Bytes: dx read once, ids, dwpe read and written (the used rows of dwte, a
    // data-dependent count, are left out)
    PROF("embedding bwd", 0, 0, 0, 0.0, (double)BT * C * 4 + (double)BT * 4 + (double)T * C * 8,
         launch_embed_bwd(c, idx, h->dres, B, T, C, V, G + h->off_wte, G + h->off_wpe, (float*)h->du));
    bucket_done(h, L + 1);   // wte, wpe
}

// -------------------------------------------------------------- generation
// Cache and scratch of the generation calls, allocated on first use.
int ensure_gen(gpt2_handle* h) {
    if (h->gen_pool) return GPT2_OK;
    const size_t es = h->bf16_mode ? 2 : 4;
    const size_t L = h->L, C = h->C, Tc = h->cfg.block_size, Bm = h->cfg.max_B;
    const size_t layer = align_up(Bm * Tc * 3 * C * es);
    const size_t part = align_up((size_t)decode_part_floats(h->cfg.max_B * h->H, (int)Tc, h->hd) * 4);
    const size_t ptrs = align_up(2 * L * sizeof(void*));
    const size_t next = align_up(Bm * 4), win = align_up((size_t)h->maxBT * 4);
    const size_t dargs = align_up(sizeof(DecodeArgs));
    const size_t cnt = align_up(Bm * h->H * sizeof(int));
    const size_t dlay = align_up(L * sizeof(DecodeLayer)), mbar = align_up(sizeof(unsigned long long));
    char* pool = nullptr;
    if (cudaMalloc((void**)&pool, L * layer + part + ptrs + next + win + dargs + cnt + dlay + mbar) != cudaSuccess) {
        cudaGetLastError();
        return fail(GPT2_ERR_OOM, "cudaMalloc of the key/value cache failed");
    }
    std::vector<void*> kv(L, nullptr);
    size_t off = 0;
    for (size_t l = 0; l < L; ++l, off += layer) kv[l] = pool + off;
    float* dec_part = (float*)(pool + off);
    off += part;
    void** layer_ptrs = (void**)(pool + off);
    off += ptrs;
    int* d_next = (int*)(pool + off);
    off += next;
    int* d_window = (int*)(pool + off);
    off += win;
    DecodeArgs* d_dec = (DecodeArgs*)(pool + off);
    off += dargs;
    int* dec_counters = (int*)(pool + off);
    off += cnt;
    DecodeLayer* dec_layers = (DecodeLayer*)(pool + off);
    off += dlay;
    unsigned long long* mega_bar = (unsigned long long*)(pool + off);
    std::vector<DecodeLayer> dl(L);
    for (size_t l = 0; l < L; ++l) {
        const LayerOff& o = h->lo[l];
        dl[l] = DecodeLayer{o.ln1w, o.ln1b, o.wqkv, o.bqkv, o.wproj, o.bproj, o.ln2w, o.ln2b, o.wfc, o.bfc,
                            o.wfcp, o.bfcp};
    }
    std::vector<void*> tab(2 * L);
    for (size_t l = 0; l < L; ++l) {
        tab[l] = h->qkv[l];
        tab[L + l] = kv[l];
    }
    // the handle takes the pool only once the pointer table is on the device
    cudaError_t e = cudaMemcpyAsync(layer_ptrs, tab.data(), tab.size() * sizeof(void*), cudaMemcpyHostToDevice,
                                    h->stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(dec_counters, 0, cnt, h->stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(mega_bar, 0, mbar, h->stream);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(dec_layers, dl.data(), L * sizeof(DecodeLayer), cudaMemcpyHostToDevice, h->stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(h->stream);
    if (e != cudaSuccess) {
        cudaFree(pool);
        return fail(GPT2_ERR_CUDA, std::string("key/value cache setup: ") + cudaGetErrorString(e));
    }
    h->gen_pool = pool;
    h->kv = kv;
    h->dec_part = dec_part;
    h->d_layer_ptrs = layer_ptrs;
    h->d_next = d_next;
    h->d_window = d_window;
    h->d_dec = d_dec;
    h->dec_counters = dec_counters;
    h->d_dec_layers = dec_layers;
    h->d_mega_bar = mega_bar;
    h->kv_B = h->kv_len = 0;
    return GPT2_OK;
}

// Forward of (B, T) tokens keeping only the last position's logits (B, V),
// then k, v of every position of every layer into cache rows 0 .. T-1.
template <typename A>
void prefill_impl(gpt2_handle* h, const int* idx, int B, int T, A* logits_out) {
    forward_impl<A>(h, idx, nullptr, B, T, logits_out, nullptr, 1.f, false, true);
    const double es = sizeof(A);
    PROF("kv cache fill", 0, 0, 0, 0.0, 2.0 * h->L * B * T * 2 * h->C * es,
         launch_kv_store(h->ctx(), (const void* const*)h->d_layer_ptrs, h->d_layer_ptrs + h->L, h->L, B, T,
                         h->cfg.block_size, h->C, (int)sizeof(A)));
}

// A decode GEMM whose operand is LN(ln.x) with (ln.w, ln.b), the LayerNorm
// computed inside the weight-streaming kernel.
template <typename A>
void gemv_ln(gpt2_handle* h, const char* site, long long w_off, int M, int N, int K, const Epilogue& ep,
             const LnIn& ln) {
    PROF(site, M, N, K, 2.0 * M * N * K, gemm_bytes(M, N, K, sizeof(A), ep) + (double)M * K * (4.0 - sizeof(A)),
         launch_gemv<A>(h->ctx(), nullptr, wop<A>(h, w_off), M, N, K, ep, ln));
}

// One new position `pos` of B sequences whose cache holds rows 0 .. pos-1:
// the blocks' forward for tok (B) at that position, its q, k, v written to
// cache row pos, attention over rows 0 .. pos, logits (B, V). With pos_dev the
// position is *pos_dev, read on the device by the embedding, the c_attn GEMM's
// output row and the attention (the host's pos then only sizes the profile).
// With at most GEMV_MAX_M rows every GEMM runs on the weight-streaming kernel
// and the LayerNorms before c_attn (after the first), c_fc and lm_head run
// inside it; the kernels are chained by programmatic dependent launch.
// The persistent one-kernel decode step; false if the shape or mode does not fit.
template <typename A>
bool decode_mega(gpt2_handle* h, const int* tok, int B, int pos, A* logits_out, const int* pos_dev) {
    if (sizeof(A) != 2 || !h->use_mega || !h->bf16_mode) return false;
    MegaDecode p = {};
    p.L = h->L;
    p.C = h->C;
    p.H = h->H;
    p.V = h->V;
    p.Tc = h->cfg.block_size;
    p.B = B;
    p.pos_now = pos;
    p.pos_dev = pos_dev;
    if (!decode_mega_plan(p, h->num_sms)) return false;
    p.P = h->params;
    p.W = h->shadow;
    p.layers = h->d_dec_layers;
    p.off_wte = h->off_wte;
    p.off_wpe = h->off_wpe;
    p.off_lnfw = h->off_lnfw;
    p.off_lnfb = h->off_lnfb;
    p.kv = h->d_layer_ptrs + h->L;
    p.resid = h->resid[0];
    p.att = (bf16*)h->att[0];
    p.fcg = (bf16*)h->fcg[0];
    p.logits = (bf16*)logits_out;
    p.tok = tok;
    p.bar = h->d_mega_bar;
    Ctx c = h->ctx();
    p.status = c.status;
    const double C = h->C, weights = 2.0 * (h->L * 12.0 * C * C + (double)h->V * C);
    PROF("decode step (one persistent kernel)", 0, 0, 0, 2.0 * B * weights / 2.0,
         weights + 2.0 * h->L * B * (pos + 1.0) * 2 * C,
         if (!launch_decode_mega(c, p)) h->host_error = "the persistent decode kernel could not be launched");
    return true;
}

template <typename A>
void decode_impl(gpt2_handle* h, const int* tok, int B, int pos, A* logits_out, const int* pos_dev = nullptr) {
    if (decode_mega<A>(h, tok, B, pos, logits_out, pos_dev)) return;
    PdlScope pdl(h);
    Ctx c = h->ctx();
    const int C = h->C, V = h->V, L = h->L, H = h->H, hd = h->hd, Tc = h->cfg.block_size;
    const long long ld_kv = 3LL * C * Tc;
    const double es = sizeof(A);
    const double ln_fwd_bytes = (double)B * C * (4 + es) + 8.0 * B;
    const int n = pos + 1;
    const bool fuse = gemv_supported(sizeof(A), B, C) && gemv_supported(sizeof(A), B, 4 * C);
    float* P = h->params;
    PROF("decode embed+ln_1", 0, 0, 0, 0.0, (double)B * C * (4 + 4 + 4 + es),
         launch_embed_ln<A>(c, tok, P + h->off_wte, P + h->off_wpe + (pos_dev ? 0 : (long long)pos * C), B, 1, C,
                            V, P + h->lo[0].ln1w, P + h->lo[0].ln1b, h->resid[0], (A*)h->ln1[0], h->ln_mean[0],
                            h->ln_rstd[0], pos_dev));
    for (int l = 0; l < L; ++l) {
        const LayerOff& o = h->lo[l];
        Epilogue e = epi(EPI_BIAS, (A*)h->kv[l] + (pos_dev ? 0 : (long long)pos * 3 * C), ld_kv);
        e.bias = P + o.bqkv;
        e.out_row_dev = pos_dev;
        e.out_row_bytes = 3LL * C * (long long)sizeof(A);
        if (fuse && l > 0) {
            LnIn ln;
            ln.x = h->resid[2 * l];
            ln.w = P + o.ln1w;
            ln.b = P + o.ln1b;
            gemv_ln<A>(h, "decode ln_1+gemm c_attn", o.wqkv, B, 3 * C, C, e, ln);
        } else {
            gemm<A>(h, "decode gemm c_attn", GEMM_NT, h->ln1[l], wop<A>(h, o.wqkv), B, 3 * C, C, e);
        }
        PROF("decode attention", 0, 0, 0, 4.0 * B * H * (double)n * hd, (double)B * n * 2 * C * es,
             launch_attention_decode<A>(c, (const A*)h->kv[l], (A*)h->att[l], h->dec_part, B, H, hd, Tc, n,
                                        pos_dev, h->dec_counters));
        e = epi(EPI_BIAS_RESID, h->resid[2 * l + 1], C);
        e.bias = P + o.bproj;
        e.resid = h->resid[2 * l];
        gemm<A>(h, "decode gemm attn.c_proj", GEMM_NT, h->att[l], wop<A>(h, o.wproj), B, C, C, e);
        e = epi(EPI_BIAS_GELU, h->fcg[l], 4 * C);
        e.out2 = h->fch[l];
        e.bias = P + o.bfc;
        if (fuse) {
            LnIn ln;
            ln.x = h->resid[2 * l + 1];
            ln.w = P + o.ln2w;
            ln.b = P + o.ln2b;
            gemv_ln<A>(h, "decode ln_2+gemm c_fc+gelu", o.wfc, B, 4 * C, C, e, ln);
        } else {
            PROF("decode layernorm", 0, 0, 0, 0.0, ln_fwd_bytes,
                 launch_layernorm_fwd<A>(c, h->resid[2 * l + 1], P + o.ln2w, P + o.ln2b, (A*)h->ln2[l],
                                         h->ln_mean[2 * l + 1], h->ln_rstd[2 * l + 1], B, C));
            gemm<A>(h, "decode gemm c_fc+gelu", GEMM_NT, h->ln2[l], wop<A>(h, o.wfc), B, 4 * C, C, e);
        }
        e = epi(EPI_BIAS_RESID, h->resid[2 * l + 2], C);
        e.bias = P + o.bfcp;
        e.resid = h->resid[2 * l + 1];
        gemm<A>(h, "decode gemm mlp.c_proj", GEMM_NT, h->fcg[l], wop<A>(h, o.wfcp), B, C, 4 * C, e);
        const bool last = (l + 1 == L);
        if (!fuse)
            PROF("decode layernorm", 0, 0, 0, 0.0, ln_fwd_bytes,
                 launch_layernorm_fwd<A>(c, h->resid[2 * l + 2], last ? P + h->off_lnfw : P + h->lo[l + 1].ln1w,
                                         last ? P + h->off_lnfb : P + h->lo[l + 1].ln1b,
                                         last ? (A*)h->lnf : (A*)h->ln1[l + 1], h->ln_mean[2 * l + 2],
                                         h->ln_rstd[2 * l + 2], B, C));
    }
    if (fuse) {
        LnIn ln;
        ln.x = h->resid[2 * L];
        ln.w = P + h->off_lnfw;
        ln.b = P + h->off_lnfb;
        gemv_ln<A>(h, "decode ln_f+gemm lm_head", h->off_wte, B, V, C, epi(EPI_STORE, logits_out, V), ln);
    } else {
        gemm<A>(h, "decode gemm lm_head", GEMM_NT, h->lnf, wop<A>(h, h->off_wte), B, V, C,
                epi(EPI_STORE, logits_out, V));
    }
}

template <typename A>
void sample_impl(gpt2_handle* h, const A* logits, int B, float temperature, int top_k, const float* u, int* next,
                 int* out, long long out_ld, int out_col, const DecodeArgs* da = nullptr) {
    PROF("sample", 0, 0, 0, 0.0, (double)B * h->V * sizeof(A),
         launch_sample<A>(h->ctx(), logits, h->V, B, h->V, temperature, top_k, u, next, out, out_ld, out_col,
                          da));
}

int check_sampling(float temperature) {
    if (!(temperature > 0.f) || !std::isfinite(temperature))
        return fail(GPT2_ERR_INVALID_ARG, "temperature must be finite and > 0");
    return GPT2_OK;
}

int read_scalars(gpt2_handle* h) {
    CK(cudaMemcpyAsync(h->h_sc, h->d_sc, sizeof(DevScalars), cudaMemcpyDeviceToHost, h->stream));
    CK(cudaStreamSynchronize(h->stream));
    CK(cudaGetLastError());
    return GPT2_OK;
}

// Reports the status bits read back by read_scalars, and clears them on the
// device once reported, so that one bad call does not fail every later one.
int status_error(gpt2_handle* h) {
    const unsigned s = h->h_sc->status;
    if (!s) return GPT2_OK;
    h->h_sc->status = 0;
    CK(cudaMemsetAsync(&h->d_sc->status, 0, sizeof(unsigned), h->stream));
    if (s & STATUS_TIMEOUT) {
        // a grid barrier left mid-way would hold a stale count
        if (h->d_mega_bar) CK(cudaMemsetAsync(h->d_mega_bar, 0, sizeof(unsigned long long), h->stream));
        return fail(GPT2_ERR_TIMEOUT, "a bounded wait inside a kernel gave up");
    }
    if (s & STATUS_BAD_TOKEN) return fail(GPT2_ERR_BAD_TOKEN, "token id or target out of range");
    return GPT2_OK;
}

int pending_error(gpt2_handle* h) {
    if (h->host_error.empty()) return GPT2_OK;
    std::string m = h->host_error;
    h->host_error.clear();
    return fail(GPT2_ERR_CUDA, m);
}

int accumulate_impl(gpt2_handle* h, const int* idx, const int* targets, int B, int T, float loss_scale) {
    if (h->bf16_mode) {
        forward_impl<bf16>(h, idx, targets, B, T, nullptr, &h->d_sc->loss_accum, loss_scale, true);
        backward_impl<bf16>(h, idx, B, T);
    } else {
        forward_impl<float>(h, idx, targets, B, T, nullptr, &h->d_sc->loss_accum, loss_scale, true);
        backward_impl<float>(h, idx, B, T);
    }
    CK(cudaGetLastError());
    return pending_error(h);
}

// Starts a gradient cycle: gradients, accumulated loss and status bits to zero.
int zero_grad_impl(gpt2_handle* h) {
    CK(cudaMemsetAsync(h->grads, 0, h->n_params * sizeof(float), h->stream));
    CK(cudaMemsetAsync(&h->d_sc->loss_accum, 0, sizeof(double), h->stream));
    CK(cudaMemsetAsync(&h->d_sc->status, 0, sizeof(unsigned), h->stream));
    return GPT2_OK;
}

// zero_grad + forward + backward of one step on the tokens in the handle's own
// buffer (idx at d_tokens, targets at d_tokens + maxBT), through the step graph
// when graphs are on and the profiler is off.
int grad_pass_impl(gpt2_handle* h, int B, int T) {
    const int* idx = h->d_tokens;
    const int* tgt = h->d_tokens + h->maxBT;
    auto eager = [&]() {
        int rc = zero_grad_impl(h);
        if (!rc) rc = accumulate_impl(h, idx, tgt, B, T, 1.f);
        return rc;
    };
    if (!h->use_graphs || h->profiling) return eager();
    if (h->graph_exec && h->graph_B == B && h->graph_T == T) {
        CK(cudaGraphLaunch(h->graph_exec, h->stream));
        h->launches += h->graph_launches;
        return GPT2_OK;
    }
    if (h->graph_B != B || h->graph_T != T) {   // first step with this shape: eager
        if (h->graph_exec) cudaGraphExecDestroy(h->graph_exec);
        h->graph_exec = nullptr;
        h->graph_B = B;
        h->graph_T = T;
        return eager();
    }
    // second step with this shape: capture on a private stream (the caller's may be
    // the legacy default stream, which cannot be captured), then launch on the caller's
    if (!h->cap_stream) CK(cudaStreamCreateWithFlags(&h->cap_stream, cudaStreamNonBlocking));
    cudaStream_t user = h->stream;
    const long long l0 = h->launches;
    CK(cudaStreamBeginCapture(h->cap_stream, cudaStreamCaptureModeThreadLocal));
    h->stream = h->cap_stream;
    h->capturing = true;
    int rc = eager();
    h->capturing = false;
    h->stream = user;
    cudaGraph_t g = nullptr;
    cudaError_t e = cudaStreamEndCapture(h->cap_stream, &g);
    if (!rc && e == cudaSuccess) e = cudaGraphInstantiate(&h->graph_exec, g, 0);
    if (g) cudaGraphDestroy(g);
    if (rc) return rc;
    if (e != cudaSuccess) {
        h->graph_exec = nullptr;
        return fail(GPT2_ERR_CUDA, std::string("step graph capture failed: ") + cudaGetErrorString(e));
    }
    h->graph_launches = h->launches - l0;
    h->launches = l0;
    CK(cudaGraphLaunch(h->graph_exec, h->stream));
    h->launches += h->graph_launches;
    return GPT2_OK;
}

int update_impl(gpt2_handle* h, float lr, float* loss_host, float* norm_host) {
    Ctx c = h->ctx();
    CK(cudaMemsetAsync(&h->d_sc->sumsq, 0, sizeof(double), h->stream));
    PROF("grad norm", 0, 0, 0, 0.0, 4.0 * h->n_params, launch_sumsq(c, h->grads, h->n_params, &h->d_sc->sumsq));
    const long long t = h->step_t + 1;
    const double bc1 = 1.0 - pow(0.9, (double)t), bc2 = 1.0 - pow(0.95, (double)t);
    const float clip = h->cfg.grad_clip > 0.f ? h->cfg.grad_clip : 1.0f;
    PROF("adamw+clip", 0, 0, 0, 0.0, (28.0 + (h->bf16_mode ? 2.0 : 0.0)) * h->n_params,
         launch_adamw(c, h->d_chunks, h->n_chunks, h->params, h->grads, h->mom1, h->mom2,
                      h->bf16_mode ? h->shadow : nullptr, &h->d_sc->sumsq, &h->d_sc->loss_accum, lr, clip,
                      (float)bc1, (float)bc2, 0.1f));
    CK(cudaGetLastError());
    int rc = read_scalars(h);
    if (rc) return rc;
    if (h->profiling) prof_collect(h);
    const double loss = h->h_sc->loss_accum, ss = h->h_sc->sumsq;
    if (loss_host) *loss_host = (float)loss;
    if (norm_host) *norm_host = (float)sqrt(ss);
    rc = status_error(h);
    if (rc) return rc;
    if (!std::isfinite(loss) || !std::isfinite(ss))
        return fail(GPT2_ERR_NONFINITE, "loss or gradient norm is not finite; update skipped");
    h->step_t = t;
    h->kv_len = 0;   // the cached k, v belong to the old weights
    return GPT2_OK;
}

// One decode step of gpt2_generate on the device arguments h->d_dec: decode at
// position d_dec->pos, the draw d_dec->step into its output slot, then d_dec
// advanced to the next position and draw. `pos` is the host's copy of the
// position (profile sizes only).
template <typename A>
void decode_step_dev(gpt2_handle* h, int B, int pos, float temperature, int top_k) {
    PdlScope pdl(h);
    A* lg = (A*)h->logits;
    decode_impl<A>(h, h->d_next, B, pos, lg, &h->d_dec->pos);
    sample_impl<A>(h, lg, B, temperature, top_k, nullptr, h->d_next, nullptr, 0, 0, h->d_dec);
    launch_decode_advance(h->ctx(), h->d_dec);
}

// decode_step_dev through its CUDA graph: eager on the first step with a
// (B, temperature, top_k), captured on the second, replayed afterwards.
template <typename A>
int decode_step_graph(gpt2_handle* h, int B, int pos, float temperature, int top_k) {
    const bool same = h->dec_B == B && h->dec_temperature == temperature && h->dec_top_k == top_k;
    if (same && h->dec_graph) {
        CK(cudaGraphLaunch(h->dec_graph, h->stream));
        h->launches += h->dec_graph_launches;
        return GPT2_OK;
    }
    if (!same || !h->dec_seen) {
        if (h->dec_graph) cudaGraphExecDestroy(h->dec_graph);
        h->dec_graph = nullptr;
        h->dec_B = B;
        h->dec_temperature = temperature;
        h->dec_top_k = top_k;
        h->dec_seen = true;
        decode_step_dev<A>(h, B, pos, temperature, top_k);
        return GPT2_OK;
    }
    if (!h->cap_stream) CK(cudaStreamCreateWithFlags(&h->cap_stream, cudaStreamNonBlocking));
    cudaStream_t user = h->stream;
    const long long l0 = h->launches;
    CK(cudaStreamBeginCapture(h->cap_stream, cudaStreamCaptureModeThreadLocal));
    h->stream = h->cap_stream;
    h->capturing = true;
    decode_step_dev<A>(h, B, pos, temperature, top_k);
    h->capturing = false;
    h->stream = user;
    cudaGraph_t g = nullptr;
    cudaError_t e = cudaStreamEndCapture(h->cap_stream, &g);
    if (h->host_error.empty() && e == cudaSuccess) e = cudaGraphInstantiate(&h->dec_graph, g, 0);
    if (g) cudaGraphDestroy(g);
    if (!h->host_error.empty()) return GPT2_OK;   // reported by the caller
    if (e != cudaSuccess) {
        h->dec_graph = nullptr;
        return fail(GPT2_ERR_CUDA, std::string("decode graph capture failed: ") + cudaGetErrorString(e));
    }
    h->dec_graph_launches = h->launches - l0;
    h->launches = l0;
    CK(cudaGraphLaunch(h->dec_graph, h->stream));
    h->launches += h->dec_graph_launches;
    return GPT2_OK;
}

template <typename A>
int generate_impl(gpt2_handle* h, const int* prompt, int B, int T0, int max_new, float temperature, int top_k,
                  const float* u, int* out) {
    const int Tb = h->cfg.block_size, Ttot = T0 + max_new;
    Ctx c = h->ctx();
    PROF("token copy", 0, 0, 0, 0.0, 8.0 * B * T0, launch_copy_tokens(c, prompt, T0, out, Ttot, B, T0));
    A* lg = (A*)h->logits;
    // decode steps on device arguments (and a graph) where every decode GEMM runs
    // on the weight-streaming kernel, whose output row can be picked on the device
    const bool dev_args = h->use_graphs && !h->profiling && gemv_supported(sizeof(A), B, h->C) &&
                          gemv_supported(sizeof(A), B, 4 * h->C);
    bool args_set = false;
    for (int s = 0; s < max_new; ++s) {
        const int n = T0 + s;   // tokens so far; the draw is token n
        if (s == 0 || n > Tb) {
            const int W = std::min(n, Tb);
            PROF("token copy", 0, 0, 0, 0.0, 8.0 * B * W,
                 launch_copy_tokens(c, out + (n - W), Ttot, h->d_window, W, B, W));
            prefill_impl<A>(h, h->d_window, B, W, lg);
            h->kv_B = B;
            h->kv_len = W;
            args_set = false;
        } else if (dev_args) {
            if (!args_set) launch_decode_set(c, h->d_dec, n - 1, s, u, out, Ttot, T0);
            args_set = true;
            const int rc = decode_step_graph<A>(h, B, n - 1, temperature, top_k);
            if (rc) return rc;
            h->kv_len = n;
            if (!h->host_error.empty()) break;
            continue;
        } else {
            decode_impl<A>(h, h->d_next, B, n - 1, lg);
            h->kv_len = n;
        }
        sample_impl<A>(h, lg, B, temperature, top_k, u + (long long)s * B, h->d_next, out, Ttot, n);
        if (!h->host_error.empty()) break;
    }
    CK(cudaGetLastError());
    return pending_error(h);
}

}  // namespace

// =============================================================== C ABI
extern "C" {

const char* gpt2_last_error(void) { return g_last_error.c_str(); }

int gpt2_create(const gpt2_config* cfg, void* stream, gpt2_handle** out) {
    g_last_error.clear();
    if (!out) return fail(GPT2_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    int rc = validate_config(cfg);
    if (rc) return rc;
    int dev = 0;
    CK(cudaGetDevice(&dev));
    cudaDeviceProp prop;
    CK(cudaGetDeviceProperties(&prop, dev));
    if (prop.major != 10)
        return fail(GPT2_ERR_UNSUPPORTED_ARCH, std::string("device is sm_") + std::to_string(prop.major) +
                                                   std::to_string(prop.minor) + ", this library is built for sm_100a");
    gpt2_handle* h = new gpt2_handle();
    h->cfg = *cfg;
    h->stream = (cudaStream_t)stream;
    h->device = dev;
    h->num_sms = prop.multiProcessorCount;
    h->bf16_mode = cfg->precision == GPT2_PRECISION_BF16;
    h->C = cfg->n_embd;
    h->L = cfg->n_layer;
    h->H = cfg->n_head;
    h->hd = cfg->n_embd / cfg->n_head;
    h->V = cfg->vocab_size;
    h->maxBT = cfg->max_B * cfg->max_T;
    if (const char* e = getenv("GPT2_B200_SIMT_GEMM")) h->use_tc_gemm = (e[0] == '0');
    if (const char* e = getenv("GPT2_B200_NO_GRAPH")) h->use_graphs = (e[0] == '0');
    if (const char* e = getenv("GPT2_B200_NO_MEGA")) h->use_mega = (e[0] == '0');
    if (const char* e = getenv("GPT2_B200_SIMT_ATTENTION")) h->use_tc_attention = (e[0] == '0');
    if (const char* e = getenv("GPT2_B200_TCGEN05_ATTENTION")) h->use_tcgen05_attention = (e[0] == '1');
    if (const char* e = getenv("GPT2_B200_TCGEN05_ATTENTION_BWD")) h->use_tcgen05_attention_bwd = (e[0] == '1');
    build_layout(h);

    auto cleanup_fail = [&](int code, const std::string& msg) {
        gpt2_destroy(h);
        return fail(code, msg);
    };
    auto dmalloc = [&](void** p, size_t bytes) -> bool {
        if (cudaMalloc(p, bytes) != cudaSuccess) {
            cudaGetLastError();
            return false;
        }
        return true;
    };
    const size_t np = (size_t)h->n_params;
    if (!dmalloc((void**)&h->params, np * 4) || !dmalloc((void**)&h->grads, np * 4) ||
        !dmalloc((void**)&h->mom1, np * 4) || !dmalloc((void**)&h->mom2, np * 4) ||
        (h->bf16_mode && !dmalloc((void**)&h->shadow, np * 2)))
        return cleanup_fail(GPT2_ERR_OOM, "cudaMalloc of parameter state failed");
    std::vector<AdamChunk> chunks = build_chunks(h);
    h->n_chunks = (int)chunks.size();
    if (!dmalloc((void**)&h->d_chunks, chunks.size() * sizeof(AdamChunk)))
        return cleanup_fail(GPT2_ERR_OOM, "cudaMalloc of chunk table failed");
    if (cudaMemcpy(h->d_chunks, chunks.data(), chunks.size() * sizeof(AdamChunk), cudaMemcpyHostToDevice) !=
        cudaSuccess)
        return cleanup_fail(GPT2_ERR_CUDA, "chunk table upload failed");

    // activation pool
    const size_t es = h->bf16_mode ? 2 : 4;
    const size_t BT = (size_t)h->maxBT, C = h->C, L = h->L, V = h->V;
    const size_t BHT = (size_t)cfg->max_B * h->H * cfg->max_T;
    std::vector<std::pair<void**, size_t>> plan;
    h->resid.assign(2 * L + 1, nullptr);
    h->ln_mean.assign(2 * L + 1, nullptr);
    h->ln_rstd.assign(2 * L + 1, nullptr);
    h->ln1.assign(L, nullptr); h->ln2.assign(L, nullptr); h->qkv.assign(L, nullptr);
    h->att.assign(L, nullptr); h->fch.assign(L, nullptr); h->fcg.assign(L, nullptr);
    h->lse.assign(L, nullptr);
    for (size_t i = 0; i < 2 * L + 1; ++i) {
        plan.push_back({(void**)&h->resid[i], BT * C * 4});
        plan.push_back({(void**)&h->ln_mean[i], BT * 4});
        plan.push_back({(void**)&h->ln_rstd[i], BT * 4});
    }
    for (size_t l = 0; l < L; ++l) {
        plan.push_back({&h->ln1[l], BT * C * es});
        plan.push_back({&h->ln2[l], BT * C * es});
        plan.push_back({&h->qkv[l], BT * 3 * C * es});
        plan.push_back({&h->att[l], BT * C * es});
        plan.push_back({&h->fch[l], BT * 4 * C * es});
        plan.push_back({&h->fcg[l], BT * 4 * C * es});
        plan.push_back({(void**)&h->lse[l], BHT * 4});
    }
    plan.push_back({&h->lnf, BT * C * es});
    plan.push_back({&h->logits, BT * V * es});
    plan.push_back({(void**)&h->dres, BT * C * 4});
    plan.push_back({&h->dres_act, BT * C * es});
    plan.push_back({&h->dtmp, BT * C * es});
    plan.push_back({&h->dO, BT * C * es});
    plan.push_back({&h->dqkv, BT * 3 * C * es});
    plan.push_back({&h->du, BT * 4 * C * es});
    plan.push_back({(void**)&h->dpre, BHT * 4});
    {
        const size_t ln_part = (size_t)ln_bwd_col_blocks((int)BT) * 3 * C;
        const size_t cs_part = (size_t)colsum_row_blocks((int)BT) * 4 * C;
        const size_t mul_part = (size_t)ceil_div((int)BT, 32) * 4 * C;   // fused colsum of the GELU backward
        const size_t att_part = (size_t)cfg->max_B * ceil_div(cfg->max_T, 32) * 3 * C;   // ... of the attention bwd
        plan.push_back({(void**)&h->red_scratch, std::max(std::max(ln_part, cs_part), std::max(mul_part, att_part)) * 4});
    }
    plan.push_back({(void**)&h->d_tokens, 2 * BT * 4});
    size_t total = 0;
    for (auto& p : plan) total += align_up(p.second);
    if (!dmalloc((void**)&h->act_pool, total)) return cleanup_fail(GPT2_ERR_OOM, "cudaMalloc of activations failed");
    size_t off = 0;
    for (auto& p : plan) {
        *p.first = h->act_pool + off;
        off += align_up(p.second);
    }
    if (!dmalloc((void**)&h->d_sc, sizeof(DevScalars))) return cleanup_fail(GPT2_ERR_OOM, "cudaMalloc failed");
    if (cudaMallocHost((void**)&h->h_sc, sizeof(DevScalars)) != cudaSuccess)
        return cleanup_fail(GPT2_ERR_OOM, "cudaMallocHost failed");
    if (cudaMemsetAsync(h->d_sc, 0, sizeof(DevScalars), h->stream) != cudaSuccess ||
        cudaMemsetAsync(h->mom1, 0, np * 4, h->stream) != cudaSuccess ||
        cudaMemsetAsync(h->mom2, 0, np * 4, h->stream) != cudaSuccess ||
        cudaMemsetAsync(h->grads, 0, np * 4, h->stream) != cudaSuccess)
        return cleanup_fail(GPT2_ERR_CUDA, "initial memset failed");
    h->launches = 0;
    rc = init_weights(h);
    if (!rc) rc = refresh_shadow(h);
    if (!rc && cudaStreamSynchronize(h->stream) != cudaSuccess) rc = fail(GPT2_ERR_CUDA, "init sync failed");
    if (rc) {
        std::string msg = g_last_error;
        return cleanup_fail(rc, msg);
    }
    *out = h;
    return GPT2_OK;
}

void gpt2_destroy(gpt2_handle* h) {
    if (!h) return;
    cudaStreamSynchronize(h->stream);
    if (h->graph_exec) cudaGraphExecDestroy(h->graph_exec);
    if (h->dec_graph) cudaGraphExecDestroy(h->dec_graph);
    if (h->cap_stream) cudaStreamDestroy(h->cap_stream);
    cudaFree(h->params);
    cudaFree(h->grads);
    cudaFree(h->mom1);
    cudaFree(h->mom2);
    cudaFree(h->shadow);
    cudaFree(h->d_chunks);
    cudaFree(h->act_pool);
    cudaFree(h->gen_pool);
    cudaFree(h->d_sc);
    if (h->h_sc) cudaFreeHost(h->h_sc);
    for (cudaEvent_t e : h->pev) cudaEventDestroy(e);
    delete h;
}

int gpt2_set_stream(gpt2_handle* h, void* stream) {
    if (!h) return fail(GPT2_ERR_INVALID_ARG, "handle is NULL");
    h->stream = (cudaStream_t)stream;
    return GPT2_OK;
}

int gpt2_num_params(const gpt2_handle* h, int64_t* n) {
    if (!h || !n) return fail(GPT2_ERR_INVALID_ARG, "NULL argument");
    *n = h->n_params;
    return GPT2_OK;
}

int gpt2_param_layout(const gpt2_handle* h, gpt2_tensor_info* out, int capacity, int* count) {
    if (!h || !count) return fail(GPT2_ERR_INVALID_ARG, "NULL argument");
    *count = (int)h->tensors.size();
    if (!out) return GPT2_OK;
    if (capacity < *count) return fail(GPT2_ERR_INVALID_ARG, "capacity smaller than the tensor count");
    for (size_t i = 0; i < h->tensors.size(); ++i) {
        const TensorRec& t = h->tensors[i];
        gpt2_tensor_info& o = out[i];
        memset(&o, 0, sizeof(o));
        strncpy(o.name, t.name.c_str(), sizeof(o.name) - 1);
        o.ndim = t.ndim;
        o.shape[0] = t.shape[0];
        o.shape[1] = t.ndim == 2 ? t.shape[1] : 0;
        o.offset = t.offset;
        o.decay = t.decay;
    }
    return GPT2_OK;
}

static int copy_flat(gpt2_handle* h, void* dst, const void* src, size_t bytes, bool to_device_buf, int on_device) {
    cudaMemcpyKind k = on_device ? cudaMemcpyDeviceToDevice
                                 : (to_device_buf ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToHost);
    CK(cudaMemcpyAsync(dst, src, bytes, k, h->stream));
    CK(cudaStreamSynchronize(h->stream));
    return GPT2_OK;
}

int gpt2_set_params(gpt2_handle* h, const float* flat, int on_device) {
    if (!h || !flat) return fail(GPT2_ERR_INVALID_ARG, "NULL argument");
    h->kv_len = 0;   // the cached k, v belong to the old weights
    int rc = copy_flat(h, h->params, flat, h->n_params * 4, true, on_device);
    if (rc) return rc;
    h->launches = 0;
    rc = refresh_shadow(h);
    if (rc) return rc;
    CK(cudaStreamSynchronize(h->stream));
    return GPT2_OK;
}

int gpt2_get_params(gpt2_handle* h, float* flat, int on_device) {
    if (!h || !flat) return fail(GPT2_ERR_INVALID_ARG, "NULL argument");
    return copy_flat(h, flat, h->params, h->n_params * 4, false, on_device);
}

int gpt2_get_grads(gpt2_handle* h, float* flat, int on_device) {
    if (!h || !flat) return fail(GPT2_ERR_INVALID_ARG, "NULL argument");
    return copy_flat(h, flat, h->grads, h->n_params * 4, false, on_device);
}

int gpt2_grads_device(gpt2_handle* h, float** grads_dev, int64_t* n) {
    if (!h || !grads_dev || !n) return fail(GPT2_ERR_INVALID_ARG, "NULL argument");
    *grads_dev = h->grads;
    *n = h->n_params;
    return GPT2_OK;
}

int gpt2_debug_activation(gpt2_handle* h, int kind, int index, int B, int T, float* out_host) {
    if (!h || !out_host) return fail(GPT2_ERR_INVALID_ARG, "NULL argument");
    int rc = check_bt(h, B, T);
    if (rc) return rc;
    const int L = h->L;
    const size_t C = h->C;
    const void* src = nullptr;
    size_t width = C;
    bool fp32 = !h->bf16_mode;
    auto in = [&](int lo, int hi) { return index >= lo && index <= hi; };
    switch (kind) {
    case GPT2_ACT_RESID:
        if (!in(0, 2 * L)) break;
        src = h->resid[index];
        fp32 = true;
        break;
    case GPT2_ACT_LN1: if (in(0, L - 1)) src = h->ln1[index]; break;
    case GPT2_ACT_QKV: if (in(0, L - 1)) { src = h->qkv[index]; width = 3 * C; } break;
    case GPT2_ACT_ATTN: if (in(0, L - 1)) src = h->att[index]; break;
    case GPT2_ACT_LN2: if (in(0, L - 1)) src = h->ln2[index]; break;
    case GPT2_ACT_GELU: if (in(0, L - 1)) { src = h->fcg[index]; width = 4 * C; } break;
    case GPT2_ACT_LNF: if (index == 0) src = h->lnf; break;
    default: break;
    }
    if (!src) return fail(GPT2_ERR_INVALID_ARG, "unknown activation kind or index out of range");
    const size_t n = (size_t)B * T * width;
    if (fp32) {
        CK(cudaMemcpyAsync(out_host, src, n * 4, cudaMemcpyDeviceToHost, h->stream));
        CK(cudaStreamSynchronize(h->stream));
        return GPT2_OK;
    }
    std::vector<uint16_t> bits(n);
    CK(cudaMemcpyAsync(bits.data(), src, n * 2, cudaMemcpyDeviceToHost, h->stream));
    CK(cudaStreamSynchronize(h->stream));
    for (size_t i = 0; i < n; ++i) {   // bf16 -> fp32 is exact: the bf16 bits are the high half
        const uint32_t w = (uint32_t)bits[i] << 16;
        memcpy(&out_host[i], &w, 4);
    }
    return GPT2_OK;
}

int gpt2_get_opt_state(gpt2_handle* h, float* m, float* v, int64_t* step, int on_device) {
    if (!h) return fail(GPT2_ERR_INVALID_ARG, "NULL handle");
    int rc = GPT2_OK;
    if (m) rc = copy_flat(h, m, h->mom1, h->n_params * 4, false, on_device);
    if (!rc && v) rc = copy_flat(h, v, h->mom2, h->n_params * 4, false, on_device);
    if (step) *step = h->step_t;
    return rc;
}

int gpt2_set_opt_state(gpt2_handle* h, const float* m, const float* v, int64_t step, int on_device) {
    if (!h || !m || !v || step < 0) return fail(GPT2_ERR_INVALID_ARG, "bad argument");
    int rc = copy_flat(h, h->mom1, m, h->n_params * 4, true, on_device);
    if (!rc) rc = copy_flat(h, h->mom2, v, h->n_params * 4, true, on_device);
    if (!rc) h->step_t = step;
    return rc;
}

int gpt2_forward(gpt2_handle* h, const int32_t* idx, const int32_t* targets, int B, int T, void* logits_dev,
                 float* loss_host) {
    if (!h || !idx) return fail(GPT2_ERR_INVALID_ARG, "NULL argument");
    int rc = check_bt(h, B, T);
    if (rc) return rc;
    h->launches = 0;
    CK(cudaMemsetAsync(&h->d_sc->fwd_loss, 0, sizeof(double), h->stream));
    if (h->bf16_mode)
        forward_impl<bf16>(h, idx, targets, B, T, (bf16*)logits_dev, &h->d_sc->fwd_loss, 1.f, false);
    else
        forward_impl<float>(h, idx, targets, B, T, (float*)logits_dev, &h->d_sc->fwd_loss, 1.f, false);
    CK(cudaGetLastError());
    rc = pending_error(h);
    if (rc) return rc;
    if (loss_host || targets) {
        rc = read_scalars(h);
        if (rc) return rc;
        if (loss_host) *loss_host = (float)h->h_sc->fwd_loss;
        return status_error(h);
    }
    return GPT2_OK;
}

int gpt2_forward_last(gpt2_handle* h, const int32_t* idx, int B, int T, void* logits_dev) {
    if (!h || !idx || !logits_dev) return fail(GPT2_ERR_INVALID_ARG, "NULL argument");
    int rc = check_bt(h, B, T);
    if (rc) return rc;
    h->launches = 0;
    if (h->bf16_mode)
        forward_impl<bf16>(h, idx, nullptr, B, T, (bf16*)logits_dev, nullptr, 1.f, false, true);
    else
        forward_impl<float>(h, idx, nullptr, B, T, (float*)logits_dev, nullptr, 1.f, false, true);
    CK(cudaGetLastError());
    rc = pending_error(h);
    if (rc) return rc;
    rc = read_scalars(h);   // synchronises; reports a bad token id
    if (rc) return rc;
    return status_error(h);
}

int gpt2_prefill(gpt2_handle* h, const int32_t* idx, int B, int T, void* logits_dev) {
    if (!h || !idx || !logits_dev) return fail(GPT2_ERR_INVALID_ARG, "NULL argument");
    int rc = check_bt(h, B, T);
    if (!rc) rc = ensure_gen(h);
    if (rc) return rc;
    h->launches = 0;
    if (h->bf16_mode)
        prefill_impl<bf16>(h, idx, B, T, (bf16*)logits_dev);
    else
        prefill_impl<float>(h, idx, B, T, (float*)logits_dev);
    CK(cudaGetLastError());
    rc = pending_error(h);
    if (rc) return rc;
    h->kv_B = B;
    h->kv_len = T;
    rc = read_scalars(h);   // synchronises; reports a bad token id
    if (rc) return rc;
    return status_error(h);
}

int gpt2_decode(gpt2_handle* h, const int32_t* tokens, int B, int pos, void* logits_dev) {
    if (!h || !tokens || !logits_dev) return fail(GPT2_ERR_INVALID_ARG, "NULL argument");
    if (!h->gen_pool || h->kv_len < 1) return fail(GPT2_ERR_INVALID_ARG, "no cache: call gpt2_prefill first");
    if (B < 1 || B > h->kv_B) return fail(GPT2_ERR_INVALID_ARG, "B must be in [1, rows of the last prefill]");
    if (pos < 1 || pos > h->kv_len || pos >= h->cfg.block_size)
        return fail(GPT2_ERR_INVALID_ARG, "pos must be in [1, cached length] and < block_size");
    h->launches = 0;
    if (h->bf16_mode)
        decode_impl<bf16>(h, tokens, B, pos, (bf16*)logits_dev);
    else
        decode_impl<float>(h, tokens, B, pos, (float*)logits_dev);
    CK(cudaGetLastError());
    int rc = pending_error(h);
    if (rc) return rc;
    h->kv_len = pos + 1;
    h->kv_B = B;   // rows B .. kv_B-1 have no entry at pos: later calls may use at most B rows
    rc = read_scalars(h);
    if (rc) return rc;
    return status_error(h);
}

int gpt2_sample(gpt2_handle* h, const void* logits_dev, int B, float temperature, int top_k, const float* u_dev,
                int32_t* next_dev) {
    if (!h || !logits_dev || !u_dev || !next_dev) return fail(GPT2_ERR_INVALID_ARG, "NULL argument");
    if (B < 1) return fail(GPT2_ERR_INVALID_ARG, "B must be >= 1");
    int rc = check_sampling(temperature);
    if (rc) return rc;
    h->launches = 0;
    if (h->bf16_mode)
        sample_impl<bf16>(h, (const bf16*)logits_dev, B, temperature, top_k, u_dev, next_dev, nullptr, 0, 0);
    else
        sample_impl<float>(h, (const float*)logits_dev, B, temperature, top_k, u_dev, next_dev, nullptr, 0, 0);
    CK(cudaGetLastError());
    return GPT2_OK;
}


int gpt2_generate(gpt2_handle* h, const int32_t* prompt, int B, int T0, int max_new_tokens, float temperature,
                  int top_k, const float* u_dev, int32_t* out_dev) {
    if (!h || !prompt || !out_dev || (max_new_tokens > 0 && !u_dev))
        return fail(GPT2_ERR_INVALID_ARG, "NULL argument");
    if (B < 1 || B > h->cfg.max_B) return fail(GPT2_ERR_INVALID_ARG, "B must be in [1, max_B]");
    if (T0 < 1 || max_new_tokens < 0) return fail(GPT2_ERR_INVALID_ARG, "need T0 >= 1 and max_new_tokens >= 0");
    int rc = check_sampling(temperature);
    if (rc) return rc;
    const int Tb = h->cfg.block_size;
    if (std::min(T0, Tb) > h->cfg.max_T || (T0 + max_new_tokens - 1 > Tb && Tb > h->cfg.max_T))
        return fail(GPT2_ERR_INVALID_ARG, "a prefill window (min(T0, block_size), or block_size once the "
                                          "sequence outgrows it) exceeds max_T");
    rc = ensure_gen(h);
    if (rc) return rc;
    h->launches = 0;
    rc = h->bf16_mode ? generate_impl<bf16>(h, prompt, B, T0, max_new_tokens, temperature, top_k, u_dev, out_dev)
                      : generate_impl<float>(h, prompt, B, T0, max_new_tokens, temperature, top_k, u_dev, out_dev);
    if (rc) return rc;
    rc = read_scalars(h);
    if (rc) return rc;
    if (h->profiling) prof_collect(h);
    return status_error(h);
}

int gpt2_zero_grad(gpt2_handle* h) {
    if (!h) return fail(GPT2_ERR_INVALID_ARG, "NULL handle");
    return zero_grad_impl(h);
}

int gpt2_accumulate(gpt2_handle* h, const int32_t* idx, const int32_t* targets, int B, int T, float loss_scale) {
    if (!h || !idx || !targets) return fail(GPT2_ERR_INVALID_ARG, "NULL argument");
    int rc = check_bt(h, B, T);
    if (rc) return rc;
    h->launches = 0;
    return accumulate_impl(h, idx, targets, B, T, loss_scale);
}

int gpt2_update(gpt2_handle* h, float lr, float* loss_host, float* grad_norm_host) {
    if (!h) return fail(GPT2_ERR_INVALID_ARG, "NULL handle");
    h->launches = 0;
    return update_impl(h, lr, loss_host, grad_norm_host);
}

int gpt2_step(gpt2_handle* h, const int32_t* idx, const int32_t* targets, int B, int T, float lr, float* loss_host,
              float* grad_norm_host) {
    if (!h || !idx || !targets) return fail(GPT2_ERR_INVALID_ARG, "NULL argument");
    int rc = check_bt(h, B, T);
    if (rc) return rc;
    const size_t n = (size_t)B * T;
    CK(cudaMemcpyAsync(h->d_tokens, idx, n * 4, cudaMemcpyDeviceToDevice, h->stream));
    CK(cudaMemcpyAsync(h->d_tokens + h->maxBT, targets, n * 4, cudaMemcpyDeviceToDevice, h->stream));
    h->launches = 0;
    rc = grad_pass_impl(h, B, T);
    if (!rc) rc = update_impl(h, lr, loss_host, grad_norm_host);
    return rc;
}

int gpt2_step_host(gpt2_handle* h, const int32_t* idx_host, const int32_t* targets_host, int B, int T, float lr,
                   float* loss_host, float* grad_norm_host) {
    if (!h || !idx_host || !targets_host) return fail(GPT2_ERR_INVALID_ARG, "NULL argument");
    int rc = check_bt(h, B, T);
    if (rc) return rc;
    const size_t n = (size_t)B * T;
    CK(cudaMemcpyAsync(h->d_tokens, idx_host, n * 4, cudaMemcpyHostToDevice, h->stream));
    CK(cudaMemcpyAsync(h->d_tokens + h->maxBT, targets_host, n * 4, cudaMemcpyHostToDevice, h->stream));
    h->launches = 0;
    rc = grad_pass_impl(h, B, T);
    if (!rc) rc = update_impl(h, lr, loss_host, grad_norm_host);
    return rc;
}

int gpt2_lr_at(int64_t step, float max_lr, float min_lr, int64_t warmup, int64_t max_steps, float* lr_out) {
    if (!lr_out || step < 0 || warmup < 1 || max_steps < warmup)
        return fail(GPT2_ERR_INVALID_ARG, "lr schedule: need step >= 0, warmup >= 1, max_steps >= warmup");
    double lr;
    if (step < warmup) {
        lr = (double)max_lr * (double)(step + 1) / (double)warmup;
    } else if (step > max_steps) {
        lr = min_lr;
    } else {
        const double f = (double)(step - warmup) / (double)std::max<int64_t>(1, max_steps - warmup);
        lr = min_lr + ((double)max_lr - min_lr) * 0.5 * (1.0 + cos(M_PI * f));
    }
    *lr_out = (float)lr;
    return GPT2_OK;
}

int gpt2_profile(gpt2_handle* h, int enable) {
    if (!h) return fail(GPT2_ERR_INVALID_ARG, "NULL handle");
    CK(cudaStreamSynchronize(h->stream));
    h->ppending.clear();
    h->pev_used = 0;
    h->psites.clear();
    h->pidx.clear();
    h->profiling = enable != 0;
    if (h->profiling && h->pev.empty()) {
        h->pev.resize(8192);
        for (auto& e : h->pev) CK(cudaEventCreate(&e));
    }
    return GPT2_OK;
}

int gpt2_profile_read(gpt2_handle* h, gpt2_kernel_stat* out, int capacity, int* count) {
    if (!h || !count) return fail(GPT2_ERR_INVALID_ARG, "NULL argument");
    CK(cudaStreamSynchronize(h->stream));
    prof_collect(h);
    *count = (int)h->psites.size();
    if (!out) return GPT2_OK;
    if (capacity < *count) return fail(GPT2_ERR_INVALID_ARG, "capacity smaller than the site count");
    for (size_t i = 0; i < h->psites.size(); ++i) {
        memset(&out[i], 0, sizeof(out[i]));
        strncpy(out[i].name, h->psites[i].name.c_str(), sizeof(out[i].name) - 1);
        out[i].launches = h->psites[i].launches;
        out[i].total_ms = h->psites[i].ms;
        out[i].flops = h->psites[i].flops;
        out[i].bytes = h->psites[i].bytes;
    }
    return GPT2_OK;
}

int gpt2_grad_buckets(const gpt2_handle* h, int64_t* offsets, int64_t* counts, int capacity, int* n) {
    if (!h || !n) return fail(GPT2_ERR_INVALID_ARG, "NULL argument");
    std::vector<std::pair<long long, long long>> b;
    grad_buckets(h, b);
    *n = (int)b.size();
    if (!offsets && !counts) return GPT2_OK;
    if (!offsets || !counts || capacity < *n) return fail(GPT2_ERR_INVALID_ARG, "need offsets, counts and capacity >= n");
    for (size_t i = 0; i < b.size(); ++i) {
        offsets[i] = b[i].first;
        counts[i] = b[i].second;
    }
    return GPT2_OK;
}

int gpt2_set_grad_events(gpt2_handle* h, void* const* events, int n) {
    if (!h) return fail(GPT2_ERR_INVALID_ARG, "NULL handle");
    if (!events || n == 0) {
        h->grad_events.clear();
        return GPT2_OK;
    }
    if (n != h->L + 2) return fail(GPT2_ERR_INVALID_ARG, "n must be the bucket count (n_layer + 2)");
    std::vector<cudaEvent_t> ev(n);
    for (int i = 0; i < n; ++i) {
        if (!events[i]) return fail(GPT2_ERR_INVALID_ARG, "NULL event");
        ev[i] = (cudaEvent_t)events[i];
    }
    h->grad_events = ev;
    return GPT2_OK;
}

int gpt2_last_launch_count(const gpt2_handle* h, int64_t* n) {
    if (!h || !n) return fail(GPT2_ERR_INVALID_ARG, "NULL argument");
    *n = h->launches;
    return GPT2_OK;
}

}  // extern "C"
