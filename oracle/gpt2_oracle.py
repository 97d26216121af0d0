"""Plain, slow CPU oracle of one GPT-2 training step, in float64.

TEST INFRASTRUCTURE ONLY. Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this module. It shares no code
with the CUDA path (the only common module is the seeded input generator,
which holds none of the model's arithmetic).

Every function writes out the plain definition the pages give, with a numpy
matmul / exp / sum as the only library steps: attention materialises the whole
T x T score matrix, the loss takes an explicit log-softmax over every
vocabulary column, and the backward pass is derived by hand from the forward.

Sources (page title, section):
  * "GPT-2 from Scratch": "The config", "Embeddings: tokens and positions",
    "CausalSelfAttention" (fused qkv, heads, causal mask, scaled dot-product,
    output projection), "The MLP and GPT-2's GELU", "The Block: pre-LN and
    residuals", "Forward: logits, and loss when targets are given",
    "Weight tying", "AdamW, and weight decay on matrices only",
    "Gradient clipping", "How to scale up" (gradient accumulation),
    "Warmup and cosine decay" (the learning-rate schedule), "A generation
    loop" (temperature, top-k, one multinomial draw per step, the context
    cropped to block_size).
  * "Let's reproduce GPT-2 (124M)" synopsis: "Matching GPT-3's optimization
    hyperparameters" (betas, eps, clip 1.0, decay on 2-D tensors only) and
    "Gradient accumulation, and the bug in getting it right".
  * "Pretraining and fine-tuning nanoGPT-124M from scratch", "Supervised
    fine-tuning" (targets of -1 are skipped by the loss).

Readings where the pages are silent or the extraction lost the formula:
  * GELU: the formula image is missing from "The MLP and GPT-2's GELU"; the
    page names the tanh approximation of Hendrycks & Gimpel and PyTorch's
    nn.GELU(approximate="tanh"), so gelu(u) = 0.5 u (1 + tanh(sqrt(2/pi)(u + 0.044715 u^3))).
  * LayerNorm: biased variance, eps = 1e-5 inside the square root (PyTorch's
    default, "Debugging checklist" item 6).
  * Padded vocabulary columns take part in the softmax (no masking).
  * Loss with ignore_index: mean over the targets != -1 of that call; if every
    target is -1 the loss and all gradients are 0.
  * Clip: coef = min(1, max_norm / (norm + 1e-6)); the reported norm is pre-clip.
  * AdamW: decoupled decay scaled by lr, bias correction on both moments,
    eps added after the square root, step counter starting at 1.
  * Sampling: the multinomial draw is an inverse CDF in vocabulary order with
    the uniform number passed in; the k-th largest is taken on the logits
    before the temperature division (same order for temperature > 0).

Pins (tests/test_oracle_pins.py): finite differences, a torch float64
autograd model plus torch's own cross_entropy / clip_grad_norm_ / AdamW,
closed forms (initial loss, CE of equal logits, AdamW step 1, clip), the
causal invariant, the T = 1 attention case, GELU identities, LN moments,
the parameter count of "Counting parameters: 124,439,808", accumulation
equivalence and single-batch overfitting; for sampling, draw frequencies
over a grid of uniforms against torch's softmax, top-1 = argmax, kept ties,
and greedy generation against the torch library model. Parity pinned for
every function.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

LN_EPS = 1e-5
ADAM_BETA1 = 0.9
ADAM_BETA2 = 0.95
ADAM_EPS = 1e-8
WEIGHT_DECAY = 0.1
GRAD_CLIP = 1.0
GELU_C = math.sqrt(2.0 / math.pi)


@dataclass(frozen=True)
class Shape:
    n_layer: int
    n_head: int
    n_embd: int
    vocab_size: int
    block_size: int


# ----------------------------------------------------------------------------
# Parameters: "GPT-2 from Scratch", "The full model" / "Weight tying".
# wte is the lm_head weight (one tensor, listed once).
# ----------------------------------------------------------------------------
def layout(s: Shape):
    C, V = s.n_embd, s.vocab_size
    names = [("wte", (V, C)), ("wpe", (s.block_size, C))]
    for l in range(s.n_layer):
        names += [
            (f"h.{l}.ln_1.weight", (C,)), (f"h.{l}.ln_1.bias", (C,)),
            (f"h.{l}.attn.c_attn.weight", (3 * C, C)), (f"h.{l}.attn.c_attn.bias", (3 * C,)),
            (f"h.{l}.attn.c_proj.weight", (C, C)), (f"h.{l}.attn.c_proj.bias", (C,)),
            (f"h.{l}.ln_2.weight", (C,)), (f"h.{l}.ln_2.bias", (C,)),
            (f"h.{l}.mlp.c_fc.weight", (4 * C, C)), (f"h.{l}.mlp.c_fc.bias", (4 * C,)),
            (f"h.{l}.mlp.c_proj.weight", (C, 4 * C)), (f"h.{l}.mlp.c_proj.bias", (C,)),
        ]
    names += [("ln_f.weight", (C,)), ("ln_f.bias", (C,))]
    return names


def unflatten(s: Shape, flat) -> dict:
    out, off = {}, 0
    for name, shp in layout(s):
        n = int(np.prod(shp))
        out[name] = np.asarray(flat[off:off + n], dtype=np.float64).reshape(shp).copy()
        off += n
    assert off == len(flat), (off, len(flat))
    return out


def flatten(s: Shape, d: dict) -> np.ndarray:
    return np.concatenate([np.asarray(d[name], dtype=np.float64).reshape(-1) for name, _ in layout(s)])


def decays(s: Shape) -> dict:
    """Weight decay applies to tensors with dim >= 2: the matrices and the two
    embeddings ("AdamW, and weight decay on matrices only")."""
    return {name: (WEIGHT_DECAY if len(shp) >= 2 else 0.0) for name, shp in layout(s)}


# ----------------------------------------------------------------------------
# Building blocks, forward and hand-derived backward.
# ----------------------------------------------------------------------------
def layer_norm(x, w, b):
    """nn.LayerNorm over the last axis: (x - mean) / sqrt(biased var + eps) * w + b."""
    mu = x.mean(axis=-1, keepdims=True)
    xc = x - mu
    var = (xc * xc).mean(axis=-1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + LN_EPS)
    xhat = xc * rstd
    return xhat * w + b, (xhat, rstd)


def layer_norm_backward(dy, saved, w):
    """Gradient of layer_norm with respect to x, w and b (rows are independent)."""
    xhat, rstd = saved
    dxhat = dy * w
    dw = (dy * xhat).reshape(-1, dy.shape[-1]).sum(axis=0)
    db = dy.reshape(-1, dy.shape[-1]).sum(axis=0)
    dx = rstd * (dxhat - dxhat.mean(axis=-1, keepdims=True)
                 - xhat * (dxhat * xhat).mean(axis=-1, keepdims=True))
    return dx, dw, db


def gelu_tanh(u):
    """GPT-2's GELU, tanh approximation ("The MLP and GPT-2's GELU")."""
    return 0.5 * u * (1.0 + np.tanh(GELU_C * (u + 0.044715 * u ** 3)))


def gelu_tanh_grad(u):
    t = np.tanh(GELU_C * (u + 0.044715 * u ** 3))
    return 0.5 * (1.0 + t) + 0.5 * u * (1.0 - t * t) * GELU_C * (1.0 + 3.0 * 0.044715 * u * u)


def linear(x, w, b=None):
    """nn.Linear with the (out, in) weight layout: x @ w.T + b."""
    y = x @ w.T
    return y if b is None else y + b


def causal_attention(q, k, v):
    """softmax(q k^T / sqrt(hd)) with -inf above the diagonal, then @ v.

    q, k, v: (B, H, T, hd). Returns y (B, H, T, hd) and the probabilities P
    (B, H, T, T) ("CausalSelfAttention", "Scaled dot-product and the output
    projection" and "The causal mask as a registered buffer").
    """
    T, hd = q.shape[-2], q.shape[-1]
    att = (q @ np.swapaxes(k, -1, -2)) / math.sqrt(hd)
    future = np.triu(np.ones((T, T), dtype=bool), k=1)
    att = np.where(future, -np.inf, att)
    att = att - att.max(axis=-1, keepdims=True)
    p = np.exp(att)
    p = p / p.sum(axis=-1, keepdims=True)
    return p @ v, p


def causal_attention_backward(dy, q, k, v, p):
    hd = q.shape[-1]
    dv = np.swapaxes(p, -1, -2) @ dy
    dp = dy @ np.swapaxes(v, -1, -2)
    ds = p * (dp - (dp * p).sum(axis=-1, keepdims=True))   # softmax Jacobian, rowwise
    dq = (ds @ k) / math.sqrt(hd)
    dk = (np.swapaxes(ds, -1, -2) @ q) / math.sqrt(hd)
    return dq, dk, dv


def cross_entropy(logits, targets):
    """F.cross_entropy(..., ignore_index=-1): mean of lse(row) - row[target] over
    the rows whose target is not -1. Returns (loss, dlogits) where dlogits is the
    gradient of that mean (softmax - onehot) / n_valid, zero on ignored rows."""
    rows = logits.reshape(-1, logits.shape[-1])
    t = targets.reshape(-1)
    valid = t != -1
    n_valid = int(valid.sum())
    m = rows.max(axis=-1, keepdims=True)
    e = np.exp(rows - m)
    s = e.sum(axis=-1, keepdims=True)
    lse = (m + np.log(s))[:, 0]
    d = e / s
    if n_valid == 0:
        return 0.0, np.zeros_like(rows).reshape(logits.shape)
    tv = np.where(valid, t, 0)
    picked = rows[np.arange(rows.shape[0]), tv]
    loss = float(((lse - picked) * valid).sum() / n_valid)
    d[np.arange(rows.shape[0]), tv] -= 1.0
    d *= (valid[:, None] / n_valid)
    return loss, d.reshape(logits.shape)


# ----------------------------------------------------------------------------
# The model ("The full model", "The Block: pre-LN and residuals").
# ----------------------------------------------------------------------------
def forward(s: Shape, P: dict, idx, targets=None):
    """Returns (loss or None, logits (B,T,V), cache). idx, targets: (B, T) ints."""
    idx = np.asarray(idx)
    B, T = idx.shape
    assert T <= s.block_size
    C, H = s.n_embd, s.n_head
    hd = C // H
    cache = {"idx": idx, "layers": []}
    x = P["wte"][idx] + P["wpe"][np.arange(T)][None, :, :]          # (B,T,C)
    for l in range(s.n_layer):
        pre = f"h.{l}."
        c = {}
        a, c["ln1"] = layer_norm(x, P[pre + "ln_1.weight"], P[pre + "ln_1.bias"])
        qkv = linear(a, P[pre + "attn.c_attn.weight"], P[pre + "attn.c_attn.bias"])
        q, k, v = qkv[..., :C], qkv[..., C:2 * C], qkv[..., 2 * C:]
        heads = lambda z: z.reshape(B, T, H, hd).transpose(0, 2, 1, 3)  # noqa: E731
        q, k, v = heads(q), heads(k), heads(v)
        y, p = causal_attention(q, k, v)
        y = y.transpose(0, 2, 1, 3).reshape(B, T, C)
        x = x + linear(y, P[pre + "attn.c_proj.weight"], P[pre + "attn.c_proj.bias"])
        m, c["ln2"] = layer_norm(x, P[pre + "ln_2.weight"], P[pre + "ln_2.bias"])
        u = linear(m, P[pre + "mlp.c_fc.weight"], P[pre + "mlp.c_fc.bias"])
        g = gelu_tanh(u)
        x = x + linear(g, P[pre + "mlp.c_proj.weight"], P[pre + "mlp.c_proj.bias"])
        c.update(a=a, q=q, k=k, v=v, p=p, y=y, m=m, u=u, g=g)
        cache["layers"].append(c)
    f, cache["lnf"] = layer_norm(x, P["ln_f.weight"], P["ln_f.bias"])
    cache["f"] = f
    logits = linear(f, P["wte"])                                      # tied lm_head
    loss = None
    if targets is not None:
        loss, dlogits = cross_entropy(logits, np.asarray(targets))
        cache["dlogits"] = dlogits
    return loss, logits, cache


def backward(s: Shape, P: dict, cache, loss_scale: float = 1.0) -> dict:
    """Exact gradient of loss_scale * loss with respect to every parameter."""
    idx = cache["idx"]
    B, T = idx.shape
    C, H = s.n_embd, s.n_head
    hd = C // H
    G = {name: np.zeros(shp) for name, shp in layout(s)}
    dlogits = cache["dlogits"] * loss_scale                           # (B,T,V)
    f = cache["f"]
    # lm_head (tied): logits = f @ wte.T
    G["wte"] += dlogits.reshape(-1, dlogits.shape[-1]).T @ f.reshape(-1, C)
    df = dlogits @ P["wte"]
    dx, G["ln_f.weight"], G["ln_f.bias"] = layer_norm_backward(df, cache["lnf"], P["ln_f.weight"])
    for l in reversed(range(s.n_layer)):
        pre = f"h.{l}."
        c = cache["layers"][l]
        # x_out = x_mid + c_proj(gelu(c_fc(ln_2(x_mid))))
        dproj = dx
        G[pre + "mlp.c_proj.weight"] += dproj.reshape(-1, C).T @ c["g"].reshape(-1, 4 * C)
        G[pre + "mlp.c_proj.bias"] += dproj.reshape(-1, C).sum(axis=0)
        dg = dproj @ P[pre + "mlp.c_proj.weight"]
        du = dg * gelu_tanh_grad(c["u"])
        G[pre + "mlp.c_fc.weight"] += du.reshape(-1, 4 * C).T @ c["m"].reshape(-1, C)
        G[pre + "mlp.c_fc.bias"] += du.reshape(-1, 4 * C).sum(axis=0)
        dm = du @ P[pre + "mlp.c_fc.weight"]
        dln, dw, db = layer_norm_backward(dm, c["ln2"], P[pre + "ln_2.weight"])
        G[pre + "ln_2.weight"] += dw
        G[pre + "ln_2.bias"] += db
        dx = dx + dln
        # x_mid = x_in + c_proj(attn(ln_1(x_in)))
        G[pre + "attn.c_proj.weight"] += dx.reshape(-1, C).T @ c["y"].reshape(-1, C)
        G[pre + "attn.c_proj.bias"] += dx.reshape(-1, C).sum(axis=0)
        dy = (dx @ P[pre + "attn.c_proj.weight"]).reshape(B, T, H, hd).transpose(0, 2, 1, 3)
        dq, dk, dv = causal_attention_backward(dy, c["q"], c["k"], c["v"], c["p"])
        merge = lambda z: z.transpose(0, 2, 1, 3).reshape(B, T, C)  # noqa: E731
        dqkv = np.concatenate([merge(dq), merge(dk), merge(dv)], axis=-1)
        G[pre + "attn.c_attn.weight"] += dqkv.reshape(-1, 3 * C).T @ c["a"].reshape(-1, C)
        G[pre + "attn.c_attn.bias"] += dqkv.reshape(-1, 3 * C).sum(axis=0)
        da = dqkv @ P[pre + "attn.c_attn.weight"]
        dln, dw, db = layer_norm_backward(da, c["ln1"], P[pre + "ln_1.weight"])
        G[pre + "ln_1.weight"] += dw
        G[pre + "ln_1.bias"] += db
        dx = dx + dln
    dwte, dwpe = embedding_backward(idx, dx, s.vocab_size, s.block_size)
    G["wte"] += dwte
    G["wpe"] += dwpe
    return G


def embedding_backward(idx, dx, V: int, block_size: int):
    """Gradient of x0 = wte[idx] + wpe[arange(T)] ("GPT-2 from Scratch",
    "Embeddings: tokens and positions"): every row of dx lands on its token's row
    of the token table (a token seen n times gets the sum of its n rows; with
    "Weight tying" this adds to the lm_head term of the same table), and position
    t gets the sum over the batch of dx[:, t]. Returns (dwte (V, C), dwpe
    (block_size, C)); rows of dwpe at t >= T are zero."""
    B, T = idx.shape
    C = dx.shape[-1]
    dwte = np.zeros((V, C))
    np.add.at(dwte, idx.reshape(-1), dx.reshape(-1, C))
    dwpe = np.zeros((block_size, C))
    dwpe[:T] = dx.sum(axis=0)
    return dwte, dwpe


# ----------------------------------------------------------------------------
# Update: "Gradient clipping" and "AdamW, and weight decay on matrices only".
# ----------------------------------------------------------------------------
def grad_norm(G: dict) -> float:
    """Global L2 norm over every unique parameter tensor (the tied wte once)."""
    return math.sqrt(sum(float((g * g).sum()) for g in G.values()))


def clip_coefficient(norm: float, max_norm: float = GRAD_CLIP) -> float:
    return min(1.0, max_norm / (norm + 1e-6))


def adamw_update(s: Shape, P: dict, G: dict, M: dict, V: dict, t: int, lr: float,
                 max_norm: float = GRAD_CLIP):
    """One clipped AdamW step. t is the 1-based step counter after increment.

    Returns the pre-clip global norm. P, M, V are updated in place."""
    norm = grad_norm(G)
    coef = clip_coefficient(norm, max_norm)
    bc1 = 1.0 - ADAM_BETA1 ** t
    bc2 = 1.0 - ADAM_BETA2 ** t
    wd = decays(s)
    for name in P:
        g = G[name] * coef
        M[name] = ADAM_BETA1 * M[name] + (1.0 - ADAM_BETA1) * g
        V[name] = ADAM_BETA2 * V[name] + (1.0 - ADAM_BETA2) * g * g
        mhat = M[name] / bc1
        vhat = V[name] / bc2
        P[name] = P[name] * (1.0 - lr * wd[name]) - lr * mhat / (np.sqrt(vhat) + ADAM_EPS)
    return norm


def zeros_like(s: Shape) -> dict:
    return {name: np.zeros(shp) for name, shp in layout(s)}


def lr_schedule(step: int, max_lr: float, min_lr: float, warmup: int, max_steps: int) -> float:
    """Learning rate at a 0-based step ("GPT-2 from Scratch", "Warmup and cosine
    decay"): a linear ramp over the first `warmup` steps, reaching
    max_lr * (step + 1) / warmup at step `step`; then a half cosine from max_lr
    at step == warmup (cos 0 = 1) down to min_lr at step == max_steps (cos pi = -1),
    the midpoint halfway; min_lr after max_steps. The decay interval counts at
    least one step."""
    if step < warmup:
        return max_lr * (step + 1) / warmup
    if step > max_steps:
        return min_lr
    frac = (step - warmup) / max(1, max_steps - warmup)
    return min_lr + (max_lr - min_lr) * 0.5 * (1.0 + np.cos(np.pi * frac))


# ----------------------------------------------------------------------------
# Sampling ("GPT-2 from Scratch", "A generation loop").
# ----------------------------------------------------------------------------
def sample_next(logits, temperature: float, top_k: int, u: float):
    """One draw from a row of last-position logits.

    The row is divided by the temperature. With top_k >= 1, every entry below
    the k-th largest (k = min(top_k, V)) becomes -inf; entries equal to the
    k-th largest stay. The kept entries go through a softmax, and one index is
    drawn from it. The draw is by inverse CDF in vocabulary order: u in
    [0, 1) is given, and the result is the first j whose cumulative probability
    (inclusive) exceeds u; if rounding leaves u at or above the last cumulative
    value, the last kept index. top_k <= 0 keeps every entry. The k-th largest
    is found on the row before the division, which orders the entries the same
    way for any temperature > 0.

    Returns (j, probs, margin): probs in vocabulary order, and margin = the
    distance from u to the nearer end of the interval [cdf[j-1], cdf[j]) that
    selected j (a decision closer than the rounding of the cumulative sums to
    an end could go either way)."""
    x = np.asarray(logits, dtype=np.float64).reshape(-1)
    V = x.shape[0]
    keep = np.ones(V, dtype=bool)
    if top_k >= 1 and top_k < V:
        kth = np.sort(x)[::-1][top_k - 1]
        keep = x >= kth
    z = np.where(keep, x / temperature, -np.inf)
    e = np.exp(z - z.max())
    probs = e / e.sum()
    cdf = np.cumsum(probs)
    over = np.nonzero(cdf > u)[0]
    j = int(over[0]) if over.size else int(np.nonzero(keep)[0][-1])
    lo = cdf[j - 1] if j > 0 else 0.0
    margin = float(min(u - lo, cdf[j] - u))
    return j, probs, margin


def generate(s: Shape, P: dict, idx, max_new_tokens: int, temperature: float, top_k: int, u):
    """The pages' generation loop: crop the running sequence to its last
    block_size tokens, run the forward, take the last position's logits, draw
    the next token (sample_next) and append it; repeat. Every step recomputes
    the whole window (no cache). u: (max_new_tokens, B) uniforms in [0, 1),
    one per drawn token. Returns (tokens (B, T0 + max_new_tokens), margins
    (max_new_tokens, B))."""
    seq = np.asarray(idx).copy()
    u = np.asarray(u, dtype=np.float64)
    B = seq.shape[0]
    margins = np.zeros((max_new_tokens, B))
    for step in range(max_new_tokens):
        cond = seq[:, -s.block_size:]
        _, logits, _ = forward(s, P, cond)
        nxt = np.zeros((B, 1), dtype=seq.dtype)
        for b in range(B):
            nxt[b, 0], _, margins[step, b] = sample_next(logits[b, -1], temperature, top_k, u[step, b])
        seq = np.concatenate([seq, nxt], axis=1)
    return seq, margins


def train_step(s: Shape, P: dict, M: dict, V: dict, t: int, idx, targets, lr: float,
               max_norm: float = GRAD_CLIP):
    """zero_grad, forward, loss, backward, clip, AdamW ("The loop").

    Returns (loss, pre-clip norm, grads). P, M, V updated in place; t is the
    step number after increment (1 for the first step)."""
    loss, _, cache = forward(s, P, idx, targets)
    G = backward(s, P, cache)
    norm = adamw_update(s, P, G, M, V, t, lr, max_norm)
    return loss, norm, G


def accumulate_grads(s: Shape, P: dict, batches, n_micro=None):
    """Gradient accumulation: each micro-batch's mean loss divided by the number
    of micro-batches before its gradient is added ("How to scale up";
    "Gradient accumulation, and the bug in getting it right"). Returns
    (mean of the micro losses, summed grads)."""
    n = n_micro or len(batches)
    G = zeros_like(s)
    total = 0.0
    for idx, tgt in batches:
        loss, _, cache = forward(s, P, idx, tgt)
        g = backward(s, P, cache, loss_scale=1.0 / n)
        for k in G:
            G[k] += g[k]
        total += loss
    return total / n, G
