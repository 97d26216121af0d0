/*
 * gpt2_kernels.h -- kernel-level C ABI of libgpt2_b200.so.
 *
 * Single operations of the training step and of generation, exposed for unit
 * tests and for callers that assemble their own step. All pointers are CUDA device pointers
 * owned by the caller; every call enqueues on `stream` (a cudaStream_t, NULL =
 * legacy default stream) and returns without synchronising. `status_dev`
 * points to one caller-owned device uint32 that kernels OR error bits into
 * (bit 0: out-of-range token, bit 1: a bounded in-kernel wait gave up).
 * Return codes are the GPT2_* codes of gpt2.h; gpt2_last_error() explains them.
 */
#ifndef GPT2_B200_KERNELS_H
#define GPT2_B200_KERNELS_H

#include <stdint.h>

#include "gpt2.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Operand layouts of C[M,N] = sum_k A(m,k) B(n,k) (row-major storage):
 *   GPT2K_NT: A [M,K], B [N,K]  -- forward of nn.Linear, y = x W^T
 *   GPT2K_NN: A [M,K], B [K,N]  -- input gradient, dx = dy W
 *   GPT2K_TN: A [K,M], B [K,N]  -- weight gradient, dW = dy^T x            */
#define GPT2K_NT 0
#define GPT2K_NN 1
#define GPT2K_TN 2

/* Epilogues ("GPT-2 from Scratch": nn.Linear bias, "The MLP and GPT-2's GELU",
 * "The Block: pre-LN and residuals"):
 *   GPT2K_EPI_STORE      out = acc                                (bf16)
 *   GPT2K_EPI_BIAS       out = acc + bias[n]                      (bf16)
 *   GPT2K_EPI_BIAS_GELU  u = acc + bias[n] rounded to bf16; out = gelu_tanh(u),
 *                        out2 = gelu_tanh'(u), the factor the backward needs (bf16)
 *   GPT2K_EPI_BIAS_RESID out = resid + acc + bias[n]              (fp32)
 *   GPT2K_EPI_MUL        out = acc * aux (the GELU backward: aux = gelu_tanh'(u)) (bf16)
 *   GPT2K_EPI_ACCUM_F32  out = beta * out + acc                   (fp32)      */
#define GPT2K_EPI_STORE 0
#define GPT2K_EPI_BIAS 1
#define GPT2K_EPI_BIAS_GELU 2
#define GPT2K_EPI_BIAS_RESID 3
#define GPT2K_EPI_MUL 4
#define GPT2K_EPI_ACCUM_F32 5

/* bf16 GEMM with fp32 accumulation and a fused epilogue.
 * A, B        : bf16 operands in the given layout.
 * out, ldo    : result matrix [M, N] with row stride ldo (elements).
 * out2        : derivative output of GPT2K_EPI_BIAS_GELU (same ldo), else NULL.
 * bias        : fp32 [N] for the BIAS* epilogues, else NULL.
 * resid       : fp32 [M, N] (stride ldo) for GPT2K_EPI_BIAS_RESID, else NULL.
 * aux         : bf16 [M, N] (stride ldo) factor for GPT2K_EPI_MUL, else NULL.
 * colsum_part : GPT2K_EPI_MUL with engine 1 only, else NULL: fp32
 *               [ceil(M / 32), N] (stride N), written with the column sums of
 *               the bf16 results over each group of 32 rows (rows g*32 ..
 *               g*32+31 below M); adding its rows gives the bias gradient of
 *               the layer whose input gradient the GEMM produces.
 * engine      : 1 = tcgen05 tensor cores (TMA + TMEM), 0 = SIMT fp32-FMA kernel.
 * Errors: INVALID_ARG (sizes < 1, unknown layout/epilogue, a required pointer
 * NULL, or engine 1 with K, N, ldo (or M for TN) not a multiple of 8, or
 * GPT2K_EPI_ACCUM_F32 with beta other than 0 or 1, or colsum_part given with
 * another epilogue or engine 0). */
int gpt2k_matmul_bf16(int layout, const void* A, const void* B, int M, int N, int K, int epilogue, void* out,
                      int64_t ldo, void* out2, const float* bias, const float* resid, const void* aux,
                      float* colsum_part, float beta, int engine, uint32_t* status_dev, void* stream);

/* Element types of activation operands. */
#define GPT2K_F32 0
#define GPT2K_BF16 1

/* Causal multi-head self-attention forward ("GPT-2 from Scratch",
 * "CausalSelfAttention": softmax(q k^T / sqrt(hd)) with future positions masked,
 * times v; "Let's reproduce GPT-2 (124M)", "FlashAttention and vocabulary
 * padding": online softmax, no T x T matrix in memory).
 * qkv  : (B, T, 3C) rows [q | k | v], C = H * hd; head h owns columns
 *        [h*hd, (h+1)*hd) of each C-wide block.
 * out  : (B, T, C), heads concatenated in head order.
 * lse  : (B, H, T) fp32 log-sum-exp of each softmax row (for the backward).
 * dtype: GPT2K_F32 or GPT2K_BF16 (qkv, out); arithmetic is fp32.
 * engine: 0 = SIMT kernel (fp32 arithmetic throughout); 1 = tensor-core flash
 *         kernel (bf16 only: mma.sync bf16 products, fp32 accumulation and
 *         softmax); 2 = tcgen05 flash kernel (bf16, hd = 64 only: TMA loads,
 *         S and P*V in tensor memory, fp32 softmax). hd must be 32 or 64; T >= 1. */
int gpt2k_attention_fwd(int dtype, const void* qkv, void* out, float* lse, int B, int T, int H, int hd,
                        int engine, uint32_t* status_dev, void* stream);

/* Backward of gpt2k_attention_fwd: dqkv (B, T, 3C) = [dq | dk | dv] from qkv,
 * out, dout (B, T, C) and lse.
 * workspace_dev: caller-owned scratch, 16-byte aligned, of the number of floats
 *         gpt2k_attention_bwd_workspace gives: B*H*T (D = rowsum(dout * out))
 *         for engines 0 and 1; for engine 2 also an fp32 (B*T, C) accumulator
 *         of dQ, which the key tiles' partial products are added into, and
 *         the persistent kernel's work-item counter. Calls sharing one
 *         workspace must not overlap on the GPU.
 * colsum_part: engine 2 only, else NULL: fp32 [B * ceil(T / 32), 3C] (stride
 *         3C); row b * ceil(T / 32) + g receives the column sums of the stored
 *         dqkv rows 32 g .. min(32 g + 31, T - 1) of sequence b. Adding its rows
 *         gives the bias gradient of the layer that produced qkv.
 * engine: 0 = SIMT kernel; 1 = mma.sync tensor-core kernels (bf16); 2 = tcgen05
 *         kernels (bf16, hd = 64: one pass per (key tile, query tile) pair
 *         computes S and dP once; dK, dV accumulate in TMEM, dQ in the fp32
 *         workspace through bulk reduce-adds, whose order of arrival decides
 *         the last bits of dq). */
/* Workspace size of gpt2k_attention_bwd in floats (into *floats). Errors:
 * INVALID_ARG for sizes < 1, hd not 32 or 64, or an unknown engine. */
int gpt2k_attention_bwd_workspace(int B, int T, int H, int hd, int engine, int64_t* floats);

int gpt2k_attention_bwd(int dtype, const void* qkv, const void* out, const void* dout, const float* lse,
                        void* dqkv, int B, int T, int H, int hd, float* workspace_dev, float* colsum_part,
                        int engine, uint32_t* status_dev, void* stream);

/* gpt2k_attention_bwd without a workspace argument, for callers that cannot
 * allocate device memory (a framework whose caching allocator owns the GPU's
 * memory, or a latency-critical loop where cudaMalloc's implicit device
 * synchronisation is not allowed). The source pages have no counterpart: this
 * is an interface variant, the arithmetic is that of gpt2k_attention_bwd.
 * Scratch: a fixed 1 MiB device array inside the library (held by every GPU
 * that loads the library until exit), so B*H*T must be <= 262144; larger
 * sizes return GPT2_ERR_INVALID_ARG. The call allocates nothing. Its first
 * call on a device, with that device current, looks up the array's device
 * address (cudaGetSymbolAddress) and caches it; make that first call before
 * any stream capture. Every call shares the array: calls that overlap on the
 * GPU race, and must not be issued. engine must be 0 (the SIMT kernels: fp32
 * arithmetic on fp32 or bf16 operands); any other engine returns
 * GPT2_ERR_INVALID_ARG. No colsum_part output. Other arguments and errors as
 * gpt2k_attention_bwd. */
int gpt2k_attention_bwd_noalloc(int dtype, const void* qkv, const void* out, const void* dout, const float* lse,
                                void* dqkv, int B, int T, int H, int hd, int engine, uint32_t* status_dev,
                                void* stream);

/* Attention of the newest position of each sequence against a key/value cache
 * ("GPT-2 from Scratch", "A generation loop" and "CausalSelfAttention": the
 * last row of causal attention, which sees every earlier position).
 * cache : (B, Tc, 3C) rows [q | k | v], C = H * hd, in dtype; row (b, j) is
 *         position j of sequence b. q is read from row n - 1, k and v from
 *         rows 0 .. n - 1 (1 <= n <= Tc).
 * out   : (B, C) in dtype, heads concatenated in head order.
 * workspace_dev: caller-owned scratch of B * H * ceil(Tc / 64) * (hd + 2)
 *         floats (the key range is split over blocks of at least 64 keys).
 * hd must be 32 or 64, C a multiple of 64. fp32 arithmetic. */
int gpt2k_attention_decode(int dtype, const void* cache, void* out, int B, int H, int hd, int Tc, int n,
                           float* workspace_dev, uint32_t* status_dev, void* stream);

/* Next-token draw on rows of logits ("GPT-2 from Scratch", "A generation
 * loop"): row r is logits[r * ld .. r * ld + V - 1] in dtype; the draw is that
 * of gpt2_sample (temperature, top-k with ties at the k-th value kept, softmax,
 * inverse CDF at u_dev[r] in vocabulary order). next_dev (rows) int32 receives
 * the indices. Errors: INVALID_ARG (unknown dtype, rows or V < 1, ld < V, a
 * NULL pointer, temperature not finite and > 0). */
int gpt2k_sample(int dtype, const void* logits, int rows, int V, int64_t ld, float temperature, int top_k,
                 const float* u_dev, int32_t* next_dev, uint32_t* status_dev, void* stream);

/* Backward of the embedding sum ("GPT-2 from Scratch", "Embeddings: tokens and
 * positions", with the token table tied to lm_head as in "Weight tying"):
 * dwte[idx[r]] += dx[r] for every row r = b * T + t, and dwpe[t] += sum_b dx[b * T + t].
 * idx (B*T) int32 ids in [0, V) (an id outside is clamped to that range, as in
 * the step, which rejects such ids before it gets here); dx fp32 [B*T, C];
 * dwte fp32 [V, C] and dwpe fp32 [T, C] are accumulated into, not overwritten.
 * workspace_dev: NULL, or at least gpt2k_embedding_bwd_workspace(...) floats.
 * With a workspace, V <= 65536, C a multiple of 4 and C <= 2048, each token's
 * rows are added in row order (per tile of 16384 rows, tiles in order), so
 * identical inputs give bit-identical results; otherwise fp32 atomics, whose
 * last bits depend on the order of arrival. dwpe's sums are in b order in both.
 * Errors: INVALID_ARG (B, T, C or V < 1, C not a multiple of 4, a NULL pointer
 * other than workspace_dev). */
int gpt2k_embedding_bwd(const int32_t* idx, const float* dx, int B, int T, int C, int V, float* dwte, float* dwpe,
                        float* workspace_dev, uint32_t* status_dev, void* stream);

/* Workspace size of gpt2k_embedding_bwd in floats (into *floats). Errors:
 * INVALID_ARG (B, T or C < 1, floats NULL). */
int gpt2k_embedding_bwd_workspace(int B, int T, int C, int64_t* floats);

#ifdef __cplusplus
}
#endif

#endif /* GPT2_B200_KERNELS_H */
