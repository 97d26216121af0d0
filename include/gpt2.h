/*
 * gpt2.h -- C ABI of the B200 GPT-2 training-step library (libgpt2_b200.so).
 *
 * One handle owns one GPT-2 model on one CUDA device: fp32 master weights,
 * fp32 gradients, fp32 AdamW moments, a bf16 copy of the weights (bf16 mode),
 * every saved activation and all workspace. All memory is allocated in
 * gpt2_create and released in gpt2_destroy; the one other call that allocates
 * is the first generation call on a handle (gpt2_prefill or gpt2_generate),
 * which allocates the key/value cache.
 *
 * What a step computes (page title, section of the source pages):
 *   forward      "GPT-2 from Scratch": "Embeddings: tokens and positions",
 *                "CausalSelfAttention", "The MLP and GPT-2's GELU",
 *                "The Block: pre-LN and residuals", "The full model"
 *                (tied lm_head: "Weight tying").
 *   loss         "Forward: logits, and loss when targets are given":
 *                mean cross-entropy over the targets that are not -1
 *                ("Pretraining and fine-tuning nanoGPT-124M from scratch",
 *                "Supervised fine-tuning": -1 targets are skipped).
 *   backward     the exact gradient of that loss.
 *   update       "Gradient clipping" (global L2 norm, clip at grad_clip) and
 *                "AdamW, and weight decay on matrices only" (betas 0.9/0.95,
 *                eps 1e-8, decay 0.1 on 2-D tensors only, lr-scaled decoupled
 *                decay, bias correction of both moments).
 *   accumulation "How to scale up" and "Let's reproduce GPT-2 (124M)",
 *                "Gradient accumulation, and the bug in getting it right":
 *                each micro-batch's mean loss is multiplied by loss_scale
 *                (1/n_micro) before its gradient is added.
 *   generation   "A generation loop": temperature, top-k, one multinomial
 *                draw per new token, the context cropped to block_size; here
 *                on a key/value cache (gpt2_prefill, gpt2_decode, gpt2_sample,
 *                gpt2_generate).
 *
 * Conventions
 *   * Every function returns GPT2_OK (0) or a negative GPT2_ERR_* code;
 *     gpt2_last_error() gives a message for the calling thread's last error.
 *   * Pointers named *_dev are CUDA device pointers owned by the caller,
 *     read or written in order on the handle's stream. Pointers named *_host
 *     are host memory (pinned or pageable) owned by the caller.
 *   * Token ids and targets are int32, row-major (B, T). A target of -1 is
 *     ignored by the loss. Ids must lie in [0, vocab_size); targets in
 *     {-1} U [0, vocab_size). An out-of-range id is clamped on the device and
 *     reported as GPT2_ERR_BAD_TOKEN by the next synchronising call.
 *   * Device-side error flags (BAD_TOKEN, TIMEOUT) are cleared once a call has
 *     reported them, and by gpt2_zero_grad (the start of a gradient cycle), so
 *     one bad call does not fail the calls after it.
 *   * One handle is used from one thread at a time; handles are independent.
 */
#ifndef GPT2_B200_H
#define GPT2_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define GPT2_OK                    0
#define GPT2_ERR_INVALID_ARG      -1  /* bad size, null pointer, T > block_size, ... */
#define GPT2_ERR_OOM              -2  /* cudaMalloc failed in gpt2_create            */
#define GPT2_ERR_CUDA             -3  /* a CUDA runtime call or kernel launch failed  */
#define GPT2_ERR_UNSUPPORTED_ARCH -4  /* the current device is not sm_100             */
#define GPT2_ERR_NONFINITE        -5  /* loss or gradient norm not finite; the update
                                         was skipped (parameters, moments and the step
                                         counter are unchanged)                         */
#define GPT2_ERR_BAD_TOKEN        -6  /* an id or target outside its range was seen   */
#define GPT2_ERR_TIMEOUT          -7  /* a bounded wait inside a kernel gave up        */

/* Arithmetic modes. */
#define GPT2_PRECISION_FP32 0  /* fp32 everywhere, fp32 FMA matmuls (no TF32)        */
#define GPT2_PRECISION_BF16 1  /* bf16 matmul/attention operands, fp32 accumulation,
                                  fp32 residual stream, LayerNorm, softmax, loss,
                                  gradients, master weights and AdamW state          */

typedef struct gpt2_config {
    int32_t n_layer;     /* number of blocks                                         */
    int32_t n_head;      /* heads; head width n_embd / n_head must be 32 or 64        */
    int32_t n_embd;      /* residual width C; a multiple of 64                        */
    int32_t vocab_size;  /* rows of wte = columns of the logits (padded, e.g. 50304)  */
    int32_t block_size;  /* rows of wpe = largest T                                   */
    int32_t max_B;       /* largest batch passed to forward/accumulate/step           */
    int32_t max_T;       /* largest sequence length (<= block_size)                   */
    int32_t precision;   /* GPT2_PRECISION_FP32 or GPT2_PRECISION_BF16                */
    uint64_t seed;       /* seed of the on-device initialisation                      */
    float grad_clip;     /* clip threshold of the global gradient norm; <= 0 means 1.0 */
    uint32_t flags;      /* reserved, must be 0                                       */
} gpt2_config;

typedef struct gpt2_tensor_info {
    char name[48];       /* e.g. "wte", "h.3.attn.c_attn.weight", "ln_f.bias"         */
    int32_t ndim;        /* 1 or 2                                                    */
    int64_t shape[2];    /* (out, in) for Linear weights, (rows, C) for embeddings    */
    int64_t offset;      /* element offset in the flat parameter vector               */
    int32_t decay;       /* 1 if AdamW applies weight decay to this tensor (ndim 2)    */
} gpt2_tensor_info;

typedef struct gpt2_handle gpt2_handle;

/* Message of the calling thread's last error ("" if none). Never NULL. */
const char* gpt2_last_error(void);

/* Create a model on the current CUDA device.
 * cfg     : sizes and mode (see gpt2_config). Copied; the caller keeps ownership.
 * stream  : cudaStream_t every later call is ordered on (NULL = legacy default).
 * out     : receives the handle.
 * Weights are initialised on the device ("GPT-2 from Scratch", "Initialization:
 * 0.02, and the residual scaling"): N(0, 0.02) for wte, wpe and the Linear
 * weights, N(0, 0.02/sqrt(2 n_layer)) for both c_proj weights, zero biases,
 * LayerNorm weight 1, bias 0. AdamW moments and the step counter start at 0.
 * Kernel choice in bf16 mode (read from the environment here, once per handle;
 * the defaults are the fastest measured):
 *   GPT2_B200_SIMT_GEMM=1             SIMT GEMMs instead of the tcgen05 ones
 *   GPT2_B200_SIMT_ATTENTION=1        SIMT attention instead of the tensor-core kernels
 *   GPT2_B200_TCGEN05_ATTENTION=0     mma.sync attention forward instead of tcgen05
 *   GPT2_B200_TCGEN05_ATTENTION_BWD=0 mma.sync attention backward instead of tcgen05
 *   GPT2_B200_NO_GRAPH=1              no CUDA-graph replay of the step (see gpt2_step)
 *                                     nor of gpt2_generate's decode steps
 *   GPT2_B200_NO_MEGA=1               decode steps as a chain of kernels instead of
 *                                     the one persistent kernel (see gpt2_decode)
 * fp32 mode always uses the SIMT kernels.
 * Errors: INVALID_ARG (sizes), UNSUPPORTED_ARCH, OOM, CUDA. */
int gpt2_create(const gpt2_config* cfg, void* stream, gpt2_handle** out);

/* Release every resource of the handle (synchronises its stream). NULL is a no-op. */
void gpt2_destroy(gpt2_handle* h);

/* Change the stream later calls are ordered on. */
int gpt2_set_stream(gpt2_handle* h, void* stream);

/* Number of parameters with the tied wte/lm_head counted once
 * ("Counting parameters: 124,439,808" at vocab 50257, 12 layers, width 768). */
int gpt2_num_params(const gpt2_handle* h, int64_t* n);

/* Ordered parameter list of the flat vector used by the get/set calls:
 * wte, wpe, h.{l}.{ln_1.weight, ln_1.bias, attn.c_attn.weight, attn.c_attn.bias,
 * attn.c_proj.weight, attn.c_proj.bias, ln_2.weight, ln_2.bias, mlp.c_fc.weight,
 * mlp.c_fc.bias, mlp.c_proj.weight, mlp.c_proj.bias}, ln_f.weight, ln_f.bias.
 * out may be NULL to query *count; otherwise it must hold capacity entries. */
int gpt2_param_layout(const gpt2_handle* h, gpt2_tensor_info* out, int capacity, int* count);

/* Copy the flat fp32 master parameters in or out (n_params floats).
 * on_device != 0: flat is a device pointer; else host memory. set also refreshes
 * the bf16 weight copy. Synchronous. */
int gpt2_set_params(gpt2_handle* h, const float* flat, int on_device);
int gpt2_get_params(gpt2_handle* h, float* flat, int on_device);
/* Accumulated fp32 gradients (after the last accumulate/step, before clipping). */
int gpt2_get_grads(gpt2_handle* h, float* flat, int on_device);
/* The handle's own flat fp32 gradient vector, in place: *grads_dev receives its
 * device address (n_params floats in gpt2_param_layout order, *n receives
 * n_params). The handle owns it until gpt2_destroy. Work on it must be ordered
 * with the handle's stream. Data parallelism uses it ("Let's reproduce GPT-2
 * (124M)", "Scaling to 8 GPUs with DistributedDataParallel"): between the
 * last gpt2_accumulate and gpt2_update, the ranks all-reduce (sum) this buffer
 * in place, each rank having scaled its losses by 1/world, so that every rank
 * clips and updates with the average gradient. Errors: INVALID_ARG (NULL). */
int gpt2_grads_device(gpt2_handle* h, float** grads_dev, int64_t* n);
/* Saved activations of the last forward, for a layer-by-layer comparison with a
 * reference (the debugging advice of the source pages: compare each layer's
 * activations, where a 1e-6 gap is rounding and a 1e-2 gap is a bug).
 * kind / index:
 *   GPT2_ACT_RESID  0..2L  residual stream (fp32): 0 = wte[idx] + wpe[t], 2l+1 =
 *                          after block l's attention, 2l+2 = after block l's MLP
 *   GPT2_ACT_LN1    0..L-1 ln_1 output of block l               (B, T, C)
 *   GPT2_ACT_QKV    0..L-1 c_attn output of block l [q | k | v]  (B, T, 3C)
 *   GPT2_ACT_ATTN   0..L-1 attention output of block l, heads concatenated, before
 *                          attn.c_proj                           (B, T, C)
 *   GPT2_ACT_LN2    0..L-1 ln_2 output of block l               (B, T, C)
 *   GPT2_ACT_GELU   0..L-1 gelu(c_fc output) of block l         (B, T, 4C)
 *   GPT2_ACT_LNF    0      ln_f output                           (B, T, C)
 * B, T: those of the last forward (gpt2_forward, gpt2_accumulate, gpt2_step or
 * gpt2_forward_last). out_host: B * T * width floats (host), receiving the values
 * widened to fp32 (exactly, from bf16 in bf16 mode). Synchronous.
 * Errors: INVALID_ARG (NULL, kind or index out of range, B or T out of range). */
#define GPT2_ACT_RESID 0
#define GPT2_ACT_LN1 1
#define GPT2_ACT_QKV 2
#define GPT2_ACT_ATTN 3
#define GPT2_ACT_LN2 4
#define GPT2_ACT_GELU 5
#define GPT2_ACT_LNF 6
int gpt2_debug_activation(gpt2_handle* h, int kind, int index, int B, int T, float* out_host);

/* AdamW state: first and second moments (n_params floats each) and the step count. */
int gpt2_get_opt_state(gpt2_handle* h, float* m, float* v, int64_t* step, int on_device);
int gpt2_set_opt_state(gpt2_handle* h, const float* m, const float* v, int64_t step, int on_device);

/* Forward pass only (no gradients, no parameter change).
 * idx_dev      : (B, T) int32 token ids on the device.
 * targets_dev  : (B, T) int32 or NULL. With targets, *loss_host receives the mean
 *                cross-entropy over targets != -1 (0 if all are -1).
 * logits_dev   : NULL or a device buffer for (B, T, vocab_size) logits: fp32 in
 *                fp32 mode, bf16 in bf16 mode.
 * loss_host    : NULL or a host float. If non-NULL the call synchronises.
 * Errors: INVALID_ARG (B > max_B, T > max_T, T > block_size, B or T < 1). */
int gpt2_forward(gpt2_handle* h, const int32_t* idx_dev, const int32_t* targets_dev,
                 int B, int T, void* logits_dev, float* loss_host);

/* Forward pass with the logits of each sequence's last position only, the
 * input of next-token sampling ("GPT-2 from Scratch", "A generation loop": the
 * forward without targets keeps only the last position's logits, from which
 * the next token is drawn).
 * The blocks and ln_f run on all T positions (causal attention needs them);
 * the tied lm_head runs on the B last rows, so no (B, T, vocab_size) tensor is
 * formed.
 * idx_dev    : (B, T) int32 token ids on the device.
 * logits_dev : device buffer for (B, vocab_size) logits: fp32 in fp32 mode,
 *              bf16 in bf16 mode; row b = position T - 1 of sequence b.
 * Synchronises once at the end. Errors: as gpt2_forward; BAD_TOKEN for an id
 * outside [0, vocab_size). */
int gpt2_forward_last(gpt2_handle* h, const int32_t* idx_dev, int B, int T, void* logits_dev);

/* ---- Generation ("GPT-2 from Scratch", "A generation loop") ----------------
 * The pages' loop recomputes the whole (cropped) sequence for every new token;
 * these calls keep each layer's k and v rows in a key/value cache instead, so
 * a new token costs one position's forward plus attention over the cached
 * rows. The results are those of the full recompute (up to rounding). The
 * cache (per layer max_B x block_size rows of 3 * n_embd elements, in the
 * precision mode's type) is allocated by the first generation call and freed
 * by gpt2_destroy. The calls reuse the handle's activation buffers: call them
 * between training calls, not between gpt2_accumulate and gpt2_update. A
 * weight change (gpt2_update, gpt2_step, gpt2_step_host, gpt2_set_params)
 * empties the cache: gpt2_decode then needs a new gpt2_prefill. */

/* Forward of (B, T) tokens as gpt2_forward_last (logits (B, vocab_size) of the
 * last positions into logits_dev), then every layer's k and v of positions
 * 0 .. T-1 into cache rows 0 .. T-1 of sequences 0 .. B-1.
 * Synchronises once at the end. Errors: as gpt2_forward_last; OOM if the cache
 * cannot be allocated. */
int gpt2_prefill(gpt2_handle* h, const int32_t* idx_dev, int B, int T, void* logits_dev);

/* One new position: tokens_dev (B) int32 on the device are the tokens at
 * position pos of sequences 0 .. B-1, whose cache rows 0 .. pos-1 hold the
 * earlier positions (a gpt2_prefill of length pos, or a prefill followed by
 * decodes at the positions up to pos - 1). Runs the blocks on the B rows at
 * position pos, writes their k and v to cache row pos, attends over rows
 * 0 .. pos, and writes the logits (B, vocab_size) (fp32 or bf16 by mode) to
 * logits_dev. Afterwards the cache holds pos + 1 positions of sequences
 * 0 .. B-1 only: later decodes may use at most B rows.
 * In bf16 mode with B <= 4 and head width 64, when each SM's slice of every
 * weight matrix fits its 36 KB shared-memory slots (GPT-2 124M; wider models
 * fall back), the step is one persistent kernel (one CTA per SM, grid
 * barriers between the phases of a layer, the bias + rounding + residual
 * arithmetic of the other engines); otherwise a chain of kernels. The two
 * agree to bf16 rounding.
 * Synchronises once at the end. Errors: INVALID_ARG (no prefill yet, B above
 * the rows of the last prefill or decode, pos < 1, pos above the cached
 * length, or pos >= block_size); BAD_TOKEN for an id outside [0, vocab_size);
 * TIMEOUT if a grid barrier of the persistent kernel gave up (bounded wait). */
int gpt2_decode(gpt2_handle* h, const int32_t* tokens_dev, int B, int pos, void* logits_dev);

/* One draw per row of logits_dev (B, vocab_size) (fp32 or bf16 by mode, rows
 * contiguous): the row divided by temperature; with 1 <= top_k < vocab_size,
 * entries below the top_k-th largest dropped (entries equal to it kept;
 * top_k <= 0 or >= vocab_size keeps all); softmax; the index drawn is the
 * first, in vocabulary order, whose cumulative probability exceeds u_dev[b]
 * (inverse CDF: u_dev holds B uniforms in [0, 1) drawn by the caller; a value
 * below 0 counts as 0, one at or above the last cumulative value gives the
 * last kept index). next_dev (B) int32 receives the indices.
 * Asynchronous. Errors: INVALID_ARG (NULL pointer, B < 1, temperature not
 * finite and > 0). The logits must be finite. */
int gpt2_sample(gpt2_handle* h, const void* logits_dev, int B, float temperature, int top_k,
                const float* u_dev, int32_t* next_dev);

/* The pages' generation loop on the device: out_dev (B, T0 + max_new_tokens)
 * int32 receives the prompt (prompt_dev (B, T0) int32) followed by
 * max_new_tokens drawn tokens. Draw s (0-based) sees the n = T0 + s tokens
 * so far: while n <= block_size the first draw runs gpt2_prefill on them and
 * later draws run gpt2_decode at position n - 1; once n > block_size each
 * draw runs gpt2_prefill on the last block_size tokens (the pages' crop, which
 * shifts every position, so the cache cannot be reused). Each draw is
 * gpt2_sample with u = u_dev[s * B + b] (u_dev: (max_new_tokens, B) floats in
 * [0, 1)). Synchronises once at the end. The decode steps read their position
 * and output slot from device memory and run as one CUDA graph per step
 * (captured once per B, temperature and top_k) unless graphs are off.
 * Errors: INVALID_ARG (NULL pointer, B outside [1, max_B], T0 < 1,
 * max_new_tokens < 0, a bad temperature, or a prefill window longer than
 * max_T: min(T0, block_size), or block_size when the sequence outgrows it);
 * OOM for the cache; BAD_TOKEN for a prompt id outside [0, vocab_size). */
int gpt2_generate(gpt2_handle* h, const int32_t* prompt_dev, int B, int T0, int max_new_tokens,
                  float temperature, int top_k, const float* u_dev, int32_t* out_dev);

/* Set every gradient to zero and clear the accumulated loss. Asynchronous. */
int gpt2_zero_grad(gpt2_handle* h);

/* Forward + loss + backward of one micro-batch; adds loss_scale x d(loss) to the
 * gradients and loss_scale x loss to the accumulated loss. Asynchronous (no
 * synchronisation, no host readback). targets_dev must not be NULL. */
int gpt2_accumulate(gpt2_handle* h, const int32_t* idx_dev, const int32_t* targets_dev,
                    int B, int T, float loss_scale);

/* Clip + AdamW on the accumulated gradients, step counter += 1.
 * loss_host / grad_norm_host (nullable host floats) receive the accumulated loss
 * and the pre-clip global gradient norm. Synchronises once at the end.
 * Returns NONFINITE if the norm or the accumulated loss is not finite, and
 * BAD_TOKEN / TIMEOUT if a micro-batch since the last gpt2_zero_grad saw an
 * out-of-range id or target, or a kernel gave up a bounded wait. In all three
 * cases the update kernel writes nothing: parameters, moments, the bf16 weight
 * copy and the step counter are unchanged. */
int gpt2_update(gpt2_handle* h, float lr, float* loss_host, float* grad_norm_host);

/* One full training step: zero_grad, accumulate(loss_scale = 1), update.
 * A step that returns NONFINITE, BAD_TOKEN or TIMEOUT leaves parameters,
 * moments and the step counter unchanged (as gpt2_update).
 * Device-resident inputs. The ids and targets are first copied (on the
 * handle's stream) into a buffer the handle owns. The first step with a given
 * (B, T) runs eagerly; the second captures its zero_grad/forward/backward
 * launches into a CUDA graph (on a private stream), and later steps with the
 * same (B, T) replay that graph on the handle's stream; the update always runs
 * eagerly. A step with another (B, T) drops the graph. The environment variable
 * GPT2_B200_NO_GRAPH=1 at gpt2_create turns graphs off; so does profiling. */
int gpt2_step(gpt2_handle* h, const int32_t* idx_dev, const int32_t* targets_dev,
              int B, int T, float lr, float* loss_host, float* grad_norm_host);

/* The same step taking HOST token buffers: the ids and targets are copied to the
 * device on the handle's stream inside the call (pinned memory gives an
 * asynchronous copy), then the step runs (graph replay as for gpt2_step) and
 * the two scalars are read back. */
int gpt2_step_host(gpt2_handle* h, const int32_t* idx_host, const int32_t* targets_host,
                   int B, int T, float lr, float* loss_host, float* grad_norm_host);

/* Learning rate for a 0-based step ("GPT-2 from Scratch", "Warmup and cosine
 * decay"; "Let's reproduce GPT-2 (124M)": 6e-4 peak, 10% floor, 715 warmup steps
 * for 124M): max_lr * (step + 1) / warmup during the first `warmup` steps, then
 * min_lr + (max_lr - min_lr) (1 + cos(pi f)) / 2 with f = (step - warmup) /
 * max(1, max_steps - warmup), and min_lr after max_steps. A host-side scalar for
 * the lr argument of gpt2_step / gpt2_update; needs no handle and no GPU.
 * Errors: INVALID_ARG (step < 0, warmup < 1, max_steps < warmup, lr_out NULL). */
int gpt2_lr_at(int64_t step, float max_lr, float min_lr, int64_t warmup, int64_t max_steps, float* lr_out);

/* Gradient buckets for the data-parallel exchange ("Let's reproduce GPT-2
 * (124M)", "Scaling to 8 GPUs with DistributedDataParallel": every process
 * averages its gradients with the others' before the update; the pages' DDP
 * overlaps that exchange with the backward). The flat gradient vector splits
 * into contiguous ranges that the backward finishes one after another: ln_f,
 * block n_layer-1, ..., block 0, then wte and wpe (the embedding backward adds
 * into the tied wte last). offsets and counts (host, capacity entries, in
 * elements of the flat vector) receive the ranges in that order and *n their
 * number, n_layer + 2. With offsets and counts NULL only *n is written.
 * Errors: INVALID_ARG (NULL handle or n, capacity below the count). */
int gpt2_grad_buckets(const gpt2_handle* h, int64_t* offsets, int64_t* counts, int capacity, int* n);

/* events: n CUDA events (cudaEvent_t, created by the caller on the handle's
 * device and owned by it) that every eager backward (gpt2_accumulate, and the
 * first step of a (B, T) in gpt2_step / gpt2_step_host) records on the handle's
 * stream, event k as soon as bucket k of gpt2_grad_buckets is final; a collective
 * on bucket k may then start on another stream while the backward continues.
 * Backwards replayed from the step graph record nothing. n must be the bucket
 * count; events NULL or n = 0 stops the recording. The events must outlive the
 * setting. Errors: INVALID_ARG (NULL handle, a wrong n, a NULL event). */
int gpt2_set_grad_events(gpt2_handle* h, void* const* events, int n);

/* Number of kernel launches the last forward/accumulate/update/step issued. */
int gpt2_last_launch_count(const gpt2_handle* h, int64_t* n);

/* Per-launch-site timing. With profiling enabled, every kernel launch site is
 * bracketed by two CUDA events on the handle's stream (device time, no host
 * synchronisation added); gpt2_profile_read synchronises and returns, per site,
 * the launch count, summed device milliseconds and the summed algorithmic
 * FLOPs and HBM bytes. gpt2_profile(h, 1) clears the statistics. */
typedef struct gpt2_kernel_stat {
    char name[96];       /* site, e.g. "gemm fwd lm_head 16384x50304x768", "classifier" */
    int64_t launches;
    double total_ms;
    double flops;        /* algorithmic floating-point operations, all launches        */
    double bytes;        /* algorithmic HBM bytes (each operand once), all launches    */
} gpt2_kernel_stat;

int gpt2_profile(gpt2_handle* h, int enable);
int gpt2_profile_read(gpt2_handle* h, gpt2_kernel_stat* out, int capacity, int* count);

#ifdef __cplusplus
}
#endif

#endif /* GPT2_B200_H */
