// Launchers of every kernel of the training step (internal C++ interface).
// Each launcher enqueues on ctx.stream and counts its launches in *ctx.launches.
#pragma once

#include "common.cuh"

namespace gpt2 {

struct Ctx {
    cudaStream_t stream;
    unsigned* status;      // device status word (STATUS_* bits)
    long long* launches;   // host counter of kernel launches
    int num_sms;
    // launch_pdl adds the programmatic stream serialisation attribute (the
    // kernels launched through it call griddep_wait in every block)
    bool pdl = false;
};

// Launch of a kernel whose blocks all call griddep_wait before they end (and
// griddep_launch): with ctx.pdl, programmatic dependent launch, so the kernel's
// blocks start, and run up to griddep_wait, while its predecessor finishes.
template <typename... KArgs, typename... Args>
inline void launch_pdl(const Ctx& ctx, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = ctx.stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = ctx.pdl ? 1 : 0;
    cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ----------------------------------------------------------------------------
// GEMM epilogues. The contraction produces fp32 acc(row, col); the epilogue
// turns it into the stored result.
// ----------------------------------------------------------------------------
enum EpiKind {
    EPI_STORE = 0,       // out[act]  = acc
    EPI_BIAS = 1,        // out[act]  = acc + bias[col]
    EPI_BIAS_GELU = 2,   // u = acc + bias[col] (rounded to act);  out[act] = gelu(u);  out2[act] = gelu'(u)
    EPI_BIAS_RESID = 3,  // out[f32]  = resid[f32] + acc + bias[col]
    EPI_MUL = 4,         // out[act]  = acc * aux[act]   (aux = the stored gelu'(u): the GELU backward)
    EPI_ACCUM_F32 = 5,   // out[f32]  = beta * out + acc
};

struct Epilogue {
    int kind = EPI_STORE;
    void* out = nullptr;
    long long ldo = 0;
    void* out2 = nullptr;          // EPI_BIAS_GELU derivative output gelu'(u) (ld = ldo)
    const float* bias = nullptr;
    const float* resid = nullptr;  // EPI_BIAS_RESID input (ld = ldo)
    const void* aux = nullptr;     // EPI_MUL factor (ld = ldo)
    float beta = 0.f;
    int split_atomic = 0;          // EPI_ACCUM_F32 partial sums of a K split: atomicAdd into out
    // EPI_MUL on the tensor-core path only: if set, per 32-row group g the
    // column sums of the bf16 results go to colsum_part[g * N + col]
    // (ceil(M / 32) x N floats); launch_colred_finalize adds them up.
    float* colsum_part = nullptr;
    // weight-streaming kernel only: if set, out moves (*out_row_dev) * out_row_bytes
    // bytes on before use (a row picked on the device, e.g. a key/value cache row)
    const int* out_row_dev = nullptr;
    long long out_row_bytes = 0;
};

// Device-resident arguments of one decode step of the generation loop, so that a
// captured step can be replayed for every position: the new token's position
// (the cache row written, the last key attended), the draw's index within the
// call, and the call's uniforms and output rows.
struct DecodeArgs {
    int pos;
    int step;
    const float* u;      // (n_draws, B) uniforms of the call
    int* out;            // (B, out_ld) token rows of the call
    long long out_ld;
    int out_col0;        // column of draw 0
};

// One decode step as one persistent kernel (bf16, head width 64, B <=
// MEGA_MAX_B rows): embedding, every block and the tied lm_head, for the
// position pos (or *pos_dev) of tokens tok (B), the cache rows written and read
// in place. Offsets are element offsets into P (fp32 parameters: LayerNorm
// weights, biases, wte and wpe for the embedding) and W (the bf16 weights).
constexpr int MEGA_MAX_B = 4;
constexpr int MEGA_MAX_L = 48;
constexpr int MEGA_SLOTS = 5;
constexpr int MEGA_SLOT_BYTES = 36 * 1024;
constexpr int MEGA_X_BYTES = 24 * 1024;   // the operand rows (B x 4C bf16 at most)
struct DecodeLayer {
    long long ln1w, ln1b, wqkv, bqkv, wproj, bproj, ln2w, ln2b, wfc, bfc, wfcp, bfcp;
};
struct MegaDecode {
    int L, C, H, V, Tc, B;
    int pos_now;                 // the position (replaced by *pos_dev if set)
    const int* pos_dev;
    const float* P;
    const bf16* W;
    const DecodeLayer* layers;   // device, L entries
    long long off_wte, off_wpe, off_lnfw, off_lnfb;
    void* const* kv;             // device, L cache pointers ((B, Tc, 3C) rows)
    float* resid;                // (B, C) fp32 residual stream
    bf16* att;                   // (B, C)
    bf16* fcg;                   // (B, 4C)
    bf16* logits;                // (B, V)
    const int* tok;              // (B)
    unsigned long long* bar;     // grid barrier count: zero before the first launch; each launch adds
                                 // 5 L x grid, so it stays a multiple of that between launches
    unsigned* status;
    // decode_mega_plan: per CTA rows of c_attn, attn.c_proj, c_fc, mlp.c_proj; the
    // lm_head rows per CTA, rows per ring chunk and chunks; the grid
    int rows[4];
    int rows_lm, chunk_lm, n_lm, grid;
};
// Fills the plan for num_sms CTAs; false if the shape does not fit (then the
// step runs as separate kernels).
bool decode_mega_plan(MegaDecode& p, int num_sms);
// false if the launch was refused (e.g. not all CTAs can be resident).
bool launch_decode_mega(const Ctx& ctx, const MegaDecode& p);

// Operand layouts of C[M,N] = sum_k A(m,k) B(n,k):
//   GEMM_NT: A row-major [M,K], B row-major [N,K]   (forward: y = x W^T)
//   GEMM_NN: A row-major [M,K], B row-major [K,N]   (dgrad:  dx = dy W)
//   GEMM_TN: A row-major [K,M], B row-major [K,N]   (wgrad:  dW = dy^T x)
enum GemmLayout { GEMM_NT = 0, GEMM_NN = 1, GEMM_TN = 2 };

// SIMT fp32-accumulating GEMM (any layout, any size). T = float or bf16 operands.
template <typename T>
void launch_gemm_simt(const Ctx& ctx, GemmLayout layout, const T* A, const T* B, int M, int N, int K,
                      const Epilogue& ep);

// Tensor-core GEMM (tcgen05 + TMEM + TMA), bf16 operands, fp32 accumulation.
// gemm_tc_supported: shape/layout constraints (16-byte row strides).
// launch_gemm_tc returns false if a tensor map could not be encoded (nothing
// is launched; the runtime reports it as an error).
bool gemm_tc_supported(GemmLayout layout, int M, int N, int K);
bool launch_gemm_tc(const Ctx& ctx, GemmLayout layout, const bf16* A, const bf16* B, int M, int N, int K,
                    const Epilogue& ep);

// Weight-streaming GEMM for M <= GEMV_MAX_M rows, NT layout only: out(m, n) =
// sum_k A[m, k] B[n, k] through the epilogue ep (every kind; epilogue_scalar's
// arithmetic). gemv_supported: the row count and 16-byte rows of A and B.
// With ln.x set, A is not read: A[m, :] = LN(ln.x[m, :]) with (ln.w, ln.b)
// (fp32 rows of K, the arithmetic of launch_layernorm_fwd), rounded to T, is
// computed in the kernel. Launched through launch_pdl.
constexpr int GEMV_MAX_M = 4;
struct LnIn {
    const float* x = nullptr;
    const float* w = nullptr;
    const float* b = nullptr;
};
bool gemv_supported(size_t elem_size, int M, int K);
template <typename T>
void launch_gemv(const Ctx& ctx, const T* A, const T* B, int M, int N, int K, const Epilogue& ep,
                 const LnIn& ln = LnIn());

// ----------------------------------------------------------------------------
// Row-wise kernels.
// ----------------------------------------------------------------------------
// x[r] = wte[idx[r]] + wpe[r % T]; then y = LN(x) with (w, b); mean/rstd saved.
// pos_dev (nullable): the wpe row of row r is *pos_dev + r % Tn.
template <typename T>
void launch_embed_ln(const Ctx& ctx, const int* idx, const float* wte, const float* wpe, int rows, int Tn, int C,
                     int V, const float* w, const float* b, float* x, T* y, float* mean, float* rstd,
                     const int* pos_dev = nullptr);
template <typename T>
void launch_layernorm_fwd(const Ctx& ctx, const float* x, const float* w, const float* b, T* y, float* mean,
                          float* rstd, int rows, int C);
// dx = LN'(x)^T dy (+ dres_in); writes dres_out (fp32) and dres_act (operand copy);
// accumulates dw += sum dy*xhat, db += sum dy and, if dbias_next != null,
// dbias_next += sum_rows dres_out. One pass over the rows writes dres and
// per-block partial column sums to scratch (ln_bwd_col_blocks(rows) x 3C
// floats) that a fixed-order finalize adds to dw, db, dbias_next. C % 4 == 0,
// C <= 2048. The block count is fixed (2 blocks on each of 148 SMs at most),
// so the summation order does not depend on the device.
inline int ln_bwd_col_blocks(int rows) { return rows < 8 * 296 ? (rows + 7) / 8 : 296; }
template <typename T>
void launch_layernorm_bwd(const Ctx& ctx, const T* dy, const float* x, const float* mean, const float* rstd,
                          const float* w, const float* dres_in, float* dres_out, T* dres_act, float* dw,
                          float* db, float* dbias_next, int rows, int C, float* scratch);

// Count targets != -1 (and flag out-of-range targets) into *n_valid.
void launch_count_targets(const Ctx& ctx, const int* targets, int n, int V, int* n_valid);
// Cross-entropy over each row of logits (in place -> dlogits * scale / n_valid);
// loss_accum (double) += scale * sum(lse - logit[target]) / n_valid.
template <typename T>
void launch_classifier(const Ctx& ctx, T* logits, const int* targets, int rows, int V, const int* n_valid,
                       float scale, double* loss_accum, int write_grad);
// dst[b, :] = src[b * Tn + Tn - 1, :] for b < B (each sequence's last row; C % 8 == 0).
template <typename T>
void launch_gather_last_rows(const Ctx& ctx, const T* src, int B, int Tn, int C, T* dst);
// Column sums: out[c] += sum_r in[r, c], through colsum_row_blocks(rows) x cols
// partials in scratch and a fixed-order finalize. cols is a multiple of 8.
inline int colsum_row_blocks(int rows) { return (rows + 31) / 32; }
template <typename T>
void launch_colsum(const Ctx& ctx, const T* in, int rows, int cols, float* out, float* scratch);
// out[j] += sum_b partial[b * n + j], b < nblk, in a fixed order.
void launch_colred_finalize(const Ctx& ctx, const float* partial, int nblk, int n, float* out);
// dwte[idx[r]] += dx[r]; dwpe[t] += sum_b dx[b, t]. With scratch (at least
// embed_bwd_scratch_floats(B * Tn, C) floats) and V <= 65536, deterministic: the
// rows of each token are added in row order (a sort by token, then sums of runs);
// otherwise per-element atomics.
inline long long embed_bwd_scratch_floats(long long rows, int C) { return rows * (long long)C + rows + 64; }
void launch_embed_bwd(const Ctx& ctx, const int* idx, const float* dx, int B, int Tn, int C, int V, float* dwte,
                      float* dwpe, float* scratch = nullptr);

// ----------------------------------------------------------------------------
// Attention (causal, per (b, h); q/k/v are column blocks of the qkv rows).
// ----------------------------------------------------------------------------
template <typename T>
void launch_attention_fwd_simt(const Ctx& ctx, const T* qkv, T* out, float* lse, int B, int Tn, int H, int hd);
template <typename T>
void launch_attention_bwd_simt(const Ctx& ctx, const T* qkv, const T* out, const T* dout, const float* lse,
                               float* dpre /* (B,H,T) scratch */, T* dqkv, int B, int Tn, int H, int hd);

// Tensor-core flash attention (mma.sync m16n8k16, bf16 operands, fp32 softmax).
void launch_attention_fwd_mma(const Ctx& ctx, const bf16* qkv, bf16* out, float* lse, int B, int Tn, int H,
                              int hd);
void launch_attention_bwd_mma(const Ctx& ctx, const bf16* qkv, const bf16* out, const bf16* dout, const float* lse,
                              float* dpre, bf16* dqkv, int B, int Tn, int H, int hd);

// tcgen05 flash attention forward (head width 64). Returns false if a tensor map
// could not be encoded (nothing launched).
bool attention_tc_supported(int hd);
bool launch_attention_fwd_tc(const Ctx& ctx, const bf16* qkv, bf16* out, float* lse, int B, int Tn, int H);
// tcgen05 flash attention backward (head width 64): a pre-pass (D = rowsum(dout *
// out) into dpre (B*H*T floats), dq_acc zeroed, *work zeroed), the fused
// persistent kernel (dK, dV into dqkv; dQ added into dq_acc, fp32 (B*T, C),
// 16-byte aligned; *work is its work-item counter) and a post-pass (dq_acc
// rounded into the dq columns of dqkv).
// colsum_part (nullable): fp32 [B * ceil(Tn / 32)][3C]; row b * ceil(Tn / 32) + g
// receives the column sums of dqkv rows 32 g .. 32 g + 31 of sequence b.
bool launch_attention_bwd_tc(const Ctx& ctx, const bf16* qkv, const bf16* out, const bf16* dout, const float* lse,
                             float* dpre, float* dq_acc, int* work, bf16* dqkv, int B, int Tn, int H,
                             float* colsum_part);
// D = rowsum(dout * out) per (b, h, t) (the backward's pre-pass).
void launch_attention_bwd_pre(const Ctx& ctx, const bf16* out, const bf16* dout, float* dpre, int B, int Tn, int H,
                              int hd);

// ----------------------------------------------------------------------------
// Generation (k_decode.cu): key/value cache rows (B, Tc, 3C) [q | k | v] per layer.
// ----------------------------------------------------------------------------
// Attention of the newest position n-1 of each sequence against cache rows
// 0 .. n-1 (q from row n-1), heads concatenated into out (B, C). The keys are
// split over `splits` blocks per (b, h) of at least DECODE_MIN_KEYS keys each
// (fewer only when n is smaller); part holds the blocks' partial softmax sums,
// decode_part_floats(B*H, Tc, hd) floats at most.
constexpr int DECODE_MIN_KEYS = 64;
inline long long decode_part_floats(int BH, int Tc, int hd) {
    return (long long)BH * ceil_div(Tc, DECODE_MIN_KEYS) * (hd + 2);
}
void attention_decode_split(int BH, int n, int num_sms, int* splits, int* chunk);
// pos_dev (nullable): n is *pos_dev + 1, read on the device (n is then ignored; the
// key range is split for n = Tc, and splits past the last key add nothing).
// counters (nullable): B*H ints, zero before the call and left zero by it; with
// them the last block of each (b, h) to finish merges the partials (one kernel),
// else a second kernel does. Launched through launch_pdl.
template <typename T>
void launch_attention_decode(const Ctx& ctx, const T* cache, T* out, float* part, int B, int H, int hd, int Tc,
                             int n, const int* pos_dev = nullptr, int* counters = nullptr);
// One draw per row of logits (row stride ld): temperature, top-k (top_k <= 0
// or >= V keeps every entry), inverse CDF at u[row] in vocabulary order.
// next[row] = the drawn index; if out != null also out[row * out_ld + out_col].
// da (nullable): u, out, out_ld and out_col are taken from *da on the device (the
// uniforms of draw da->step, column da->out_col0 + da->step).
template <typename T>
void launch_sample(const Ctx& ctx, const T* logits, long long ld, int rows, int V, float temperature, int top_k,
                   const float* u, int* next, int* out, long long out_ld, int out_col,
                   const DecodeArgs* da = nullptr);
// *da = {pos, step, u, out, out_ld, out_col0} (one thread), and its advance to the
// next position and draw (pos + 1, step + 1).
void launch_decode_set(const Ctx& ctx, DecodeArgs* da, int pos, int step, const float* u, int* out,
                       long long out_ld, int out_col0);
void launch_decode_advance(const Ctx& ctx, DecodeArgs* da);
// k, v columns of qkv rows (b * Tn + t) of every layer -> cache rows (b, t).
// qkv_ptrs, cache_ptrs: device arrays of L pointers.
void launch_kv_store(const Ctx& ctx, const void* const* qkv_ptrs, void* const* cache_ptrs, int L, int B, int Tn,
                     int Tc, int C, int elem_size);
// dst[r * dst_ld + c] = src[r * src_ld + c] for r < rows, c < cols (int32 tokens).
void launch_copy_tokens(const Ctx& ctx, const int* src, long long src_ld, int* dst, long long dst_ld, int rows,
                        int cols);

// ----------------------------------------------------------------------------
// Optimiser and parameter utilities.
// ----------------------------------------------------------------------------
struct AdamChunk {        // a run of elements inside one tensor
    long long start;
    int count;
    int decay;
};
void launch_sumsq(const Ctx& ctx, const float* g, long long n, double* out);
// Clip + AdamW over all chunks. Skips the whole update (nothing written) when
// *ctx.status has STATUS_BAD_TOKEN or STATUS_TIMEOUT set, or when *sumsq or
// *loss_accum is not finite.
void launch_adamw(const Ctx& ctx, const AdamChunk* chunks, int n_chunks, float* p, const float* g, float* m,
                  float* v, bf16* shadow, const double* sumsq, const double* loss_accum, float lr, float clip,
                  float bc1, float bc2, float wd);
void launch_to_bf16(const Ctx& ctx, const float* in, bf16* out, long long n);
// Normal(0, std) fill from a counter-based generator (Philox4x32-10) keyed by seed.
void launch_fill_normal(const Ctx& ctx, float* p, long long n, float std, unsigned long long seed,
                        unsigned long long stream_id);
void launch_fill_const(const Ctx& ctx, float* p, long long n, float value);

}  // namespace gpt2
