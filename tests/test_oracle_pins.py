"""Pins of the CPU oracle to facts other than itself (no GPU needed).

Each test checks the oracle against something the pages or the mathematics
fix: printed values (tests/golden/pages_values.json), closed forms, invariants,
finite differences, and independent library routines (torch's nn.LayerNorm,
scaled_dot_product_attention, nn.GELU(approximate="tanh"), F.cross_entropy,
clip_grad_norm_ and torch.optim.AdamW, with gradients from autograd).
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import gpt2_oracle as O
from decoder_only_transformer_sm_b200 import synthetic as S

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_values.json")))

TINY = O.Shape(n_layer=2, n_head=4, n_embd=128, vocab_size=1024, block_size=64)
MICRO = O.Shape(n_layer=2, n_head=2, n_embd=16, vocab_size=64, block_size=8)


def _syn(s: O.Shape):
    return S.ModelShape(s.n_layer, s.n_head, s.n_embd, s.vocab_size, s.block_size)


def _params(s, seed=0, kind="init"):
    flat = S.init_params(_syn(s), seed) if kind == "init" else S.random_params(_syn(s), seed)
    return O.unflatten(s, flat.astype(np.float64))


# ----------------------------------------------------------------------------
# Shapes and parameter count ("Counting parameters: 124,439,808").
# ----------------------------------------------------------------------------
def test_param_count_matches_pages():
    s = O.Shape(12, 12, 768, 50257, 1024)
    n = sum(int(np.prod(shp)) for _, shp in O.layout(s))
    assert n == GOLDEN["param_count_124M_tied"]["value"]
    # untied lm_head would add exactly V*C
    assert 50257 * 768 == GOLDEN["tie_delta"]["value"]
    # the mask buffers (one T_max x T_max per layer) are not parameters
    assert 12 * 1024 * 1024 == GOLDEN["mask_buffer_delta"]["value"]
    assert 12 * 768 ** 2 == GOLDEN["per_block_weights_124M"]["value"]


def test_layout_agrees_with_generator_layout():
    for s in (TINY, O.Shape(12, 12, 768, 50304, 1024)):
        a = [(n, tuple(shp)) for n, shp in O.layout(s)]
        b = [(n, tuple(shp)) for n, shp, _ in S.param_layout(_syn(s))]
        assert a == b


def test_debug_shapes():
    g = GOLDEN["debug_shapes"]
    s = O.Shape(1, 12, 768, 50257, 1024)   # one block is enough for the shapes
    rng = np.random.default_rng(0)
    P = {name: rng.normal(0, 0.02, shp) for name, shp in O.layout(s)}
    idx = rng.integers(0, 50257, (2, 5))
    _, logits, cache = O.forward(s, P, idx)
    assert list(logits.shape) == g["logits"]
    assert list(cache["f"].shape) == g["residual"]
    assert list(cache["layers"][0]["p"].shape) == g["scores"]


def test_resid_init_std():
    assert round(0.02 / math.sqrt(2 * 12), 4) == GOLDEN["resid_init_std_12_layers"]["value"]
    flat = S.init_params(_syn(O.Shape(12, 12, 768, 50304, 1024)), seed=3)
    P = O.unflatten(O.Shape(12, 12, 768, 50304, 1024), flat)
    w = P["h.5.mlp.c_proj.weight"]
    assert abs(w.std() - 0.02 / math.sqrt(24)) < 2e-5
    assert abs(P["h.5.mlp.c_fc.weight"].std() - 0.02) < 5e-5
    assert np.all(P["h.5.ln_1.weight"] == 1) and np.all(P["h.5.attn.c_attn.bias"] == 0)


# ----------------------------------------------------------------------------
# Initial loss ~ ln V ("Debugging checklist" item 2).
# E[loss] ~ ln V + Var(logit)/2 with Var(logit) = 0.02^2 * C for unit-variance LN rows.
# ----------------------------------------------------------------------------
def test_initial_loss_tiny():
    P = _params(TINY, seed=0)
    idx, tgt = S.uniform_tokens(4, 64, 1024, seed=1000)
    loss, _, _ = O.forward(TINY, P, idx, tgt)
    closed = math.log(1024) + 0.5 * 0.02 ** 2 * 128
    assert abs(loss - closed) < 0.05, (loss, closed)


@pytest.mark.slow
def test_initial_loss_124M_padded():
    s = O.Shape(12, 12, 768, 50304, 1024)
    P = O.unflatten(s, S.init_params(_syn(s), seed=0))
    idx, tgt = S.zipf_tokens(1, 256, 50257, seed=1001)
    loss, _, _ = O.forward(s, P, idx, tgt)
    assert abs(loss - GOLDEN["init_loss_V50304"]["value"]) < 0.2
    assert abs(loss - (math.log(50304) + 0.5 * 0.02 ** 2 * 768)) < 0.1


# ----------------------------------------------------------------------------
# Attention ("Debugging checklist" item 3; causal mask section).
# ----------------------------------------------------------------------------
def test_attention_rows_and_future():
    rng = np.random.default_rng(1)
    q, k, v = (rng.normal(size=(2, 3, 17, 8)) for _ in range(3))
    y, p = O.causal_attention(q, k, v)
    assert np.allclose(p.sum(-1), 1.0, atol=1e-12)
    assert np.all(p[..., np.triu_indices(17, 1)[0], np.triu_indices(17, 1)[1]] == 0.0)
    # brute force, one (b, h, i) at a time
    for (b, h, i) in [(0, 0, 0), (1, 2, 16), (0, 1, 7)]:
        s = np.array([q[b, h, i] @ k[b, h, j] / math.sqrt(8) for j in range(i + 1)])
        w = np.exp(s - s.max()); w /= w.sum()
        assert np.allclose(y[b, h, i], (w[:, None] * v[b, h, :i + 1]).sum(0), atol=1e-12)


def test_attention_T1_is_v():
    rng = np.random.default_rng(2)
    q, k, v = (rng.normal(size=(2, 3, 1, 8)) for _ in range(3))
    y, _ = O.causal_attention(q, k, v)
    assert np.array_equal(y, v)


def test_causal_invariance():
    P = _params(TINY, seed=4, kind="random")
    idx, _ = S.uniform_tokens(2, 40, 1024, seed=5)
    _, la, _ = O.forward(TINY, P, idx)
    idx2 = idx.copy()
    t = 17
    idx2[:, t + 1:] = (idx2[:, t + 1:] + 123) % 1024
    _, lb, _ = O.forward(TINY, P, idx2)
    assert np.array_equal(la[:, :t + 1], lb[:, :t + 1])
    assert not np.allclose(la[:, t + 1:], lb[:, t + 1:])


def test_position_zero_indexing():
    """Row t uses wpe[t] (positions start at 0): changing wpe[7] moves only position 7.

    The perturbation is random, since a constant shift of a row is removed by LayerNorm."""
    P = _params(TINY, seed=6, kind="random")
    idx, _ = S.uniform_tokens(1, 8, 1024, seed=7)
    _, la, _ = O.forward(TINY, P, idx)
    P["wpe"][7] += np.random.default_rng(0).normal(size=128)   # last used position
    _, lb, _ = O.forward(TINY, P, idx)
    assert np.array_equal(la[:, :7], lb[:, :7]) and not np.allclose(la[:, 7], lb[:, 7])


def test_embedding_backward_is_the_transposed_jacobian():
    """x0[b, t] = wte[idx[b, t]] + wpe[t] is linear in both tables, so the gradient
    of sum(x0 * dx) is the transposed selection matrix applied to dx: one-hot(idx)^T
    dx for wte (repeated ids add up, unused ids stay zero) and, for wpe, the sum
    over b at each used position. Also a hand-worked case with a repeated id."""
    rng = np.random.default_rng(11)
    B, T, V, C, bs = 3, 5, 7, 4, 8
    idx = rng.integers(0, V, size=(B, T))
    idx[0, 0] = idx[2, 4] = 3                       # a repeat across sequences
    dx = rng.normal(size=(B, T, C))
    dwte, dwpe = O.embedding_backward(idx, dx, V, bs)
    onehot = np.zeros((B * T, V))
    onehot[np.arange(B * T), idx.reshape(-1)] = 1.0
    np.testing.assert_allclose(dwte, onehot.T @ dx.reshape(-1, C), rtol=0, atol=1e-12)
    sel = np.zeros((B * T, bs))
    sel[np.arange(B * T), np.tile(np.arange(T), B)] = 1.0
    np.testing.assert_allclose(dwpe, sel.T @ dx.reshape(-1, C), rtol=0, atol=1e-12)
    assert not dwpe[T:].any()
    small = np.array([[1, 0, 1]])
    d = np.array([[[1.0, 2.0], [3.0, 4.0], [5.0, 6.0]]])
    w, p = O.embedding_backward(small, d, 3, 4)
    assert np.array_equal(w, [[3.0, 4.0], [6.0, 8.0], [0.0, 0.0]])
    assert np.array_equal(p, [[1.0, 2.0], [3.0, 4.0], [5.0, 6.0], [0.0, 0.0]])


# ----------------------------------------------------------------------------
# GELU ("The MLP and GPT-2's GELU").
# ----------------------------------------------------------------------------
def test_gelu_identities():
    x = np.linspace(-12, 12, 200001)
    assert O.gelu_tanh(np.array([0.0]))[0] == 0.0
    assert np.max(np.abs(O.gelu_tanh(x) - O.gelu_tanh(-x) - x)) < 1e-13
    erf_gelu = 0.5 * x * (1 + np.vectorize(math.erf)(x / math.sqrt(2)))
    d = np.max(np.abs(O.gelu_tanh(x) - erf_gelu))
    assert d < GOLDEN["gelu_tanh_vs_erf_bound"]["value"] and d > 1e-5
    h = 1e-6
    fd = (O.gelu_tanh(x + h) - O.gelu_tanh(x - h)) / (2 * h)
    assert np.max(np.abs(fd - O.gelu_tanh_grad(x))) < 1e-8
    # torch's own tanh-GELU as a library routine
    torch = pytest.importorskip("torch")
    t = torch.nn.functional.gelu(torch.from_numpy(x), approximate="tanh").numpy()
    assert np.max(np.abs(t - O.gelu_tanh(x))) < 1e-14


# ----------------------------------------------------------------------------
# LayerNorm moments (biased variance, eps inside the sqrt).
# ----------------------------------------------------------------------------
def test_layernorm_moments():
    rng = np.random.default_rng(8)
    x = rng.normal(3.0, 0.01, size=(5, 64))
    y, _ = O.layer_norm(x, np.ones(64), np.zeros(64))
    var = x.var(axis=-1)
    assert np.allclose(y.mean(-1), 0.0, atol=1e-12)
    assert np.allclose((y * y).mean(-1), var / (var + O.LN_EPS), rtol=1e-12)
    b = rng.normal(size=64)
    y2, _ = O.layer_norm(x, np.ones(64), b)
    assert np.allclose(y2.mean(-1), b.mean(), atol=1e-12)


# ----------------------------------------------------------------------------
# Cross-entropy with ignore_index = -1.
# ----------------------------------------------------------------------------
def test_cross_entropy_closed_forms():
    V = 37
    logits = np.full((2, 3, V), 0.7)
    tg = np.array([[1, -1, 5], [36, 0, -1]])
    loss, d = O.cross_entropy(logits, tg)
    assert abs(loss - math.log(V)) < 1e-14
    nv = 4
    expect = np.full((2, 3, V), 1.0 / V / nv)
    expect[1 - 1 + 0, 1] = 0; expect[1, 2] = 0
    for (b, t) in [(0, 0), (0, 2), (1, 0), (1, 1)]:
        expect[b, t, tg[b, t]] -= 1.0 / nv
    assert np.allclose(d, expect, atol=1e-15)
    # all ignored
    loss0, d0 = O.cross_entropy(logits, np.full((2, 3), -1))
    assert loss0 == 0.0 and not d0.any()


def test_cross_entropy_vs_torch():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(9)
    logits = rng.normal(size=(50, 77)) * 3
    tg = rng.integers(-1, 77, size=50)
    loss, d = O.cross_entropy(logits, tg)
    lt = torch.tensor(logits, requires_grad=True)
    ref = torch.nn.functional.cross_entropy(lt, torch.tensor(tg), ignore_index=-1)
    ref.backward()
    assert abs(loss - ref.item()) < 1e-13
    assert np.max(np.abs(d - lt.grad.numpy())) < 1e-15


# ----------------------------------------------------------------------------
# Finite differences of the whole loss (double precision).
# ----------------------------------------------------------------------------
def _fd_check(s, P, idx, tgt, coords_per_tensor, rng, h=1e-5):
    loss, _, cache = O.forward(s, P, idx, tgt)
    G = O.backward(s, P, cache)
    for name, shp in O.layout(s):
        n = int(np.prod(shp))
        picks = np.arange(n) if coords_per_tensor is None or n <= coords_per_tensor \
            else rng.choice(n, coords_per_tensor, replace=False)
        flatp = P[name].reshape(-1)
        g = G[name].reshape(-1)
        for i in picks:
            old = flatp[i]
            flatp[i] = old + h
            lp, _, _ = O.forward(s, P, idx, tgt)
            flatp[i] = old - h
            lm, _, _ = O.forward(s, P, idx, tgt)
            flatp[i] = old
            fd = (lp - lm) / (2 * h)
            assert abs(fd - g[i]) <= 1e-5 * abs(g[i]) + 2e-9, (name, i, fd, g[i])


def test_finite_differences_micro_every_coordinate():
    s = MICRO
    P = _params(s, seed=10, kind="random")
    for k in P:                                   # larger weights: stronger nonlinearity
        if k.endswith(".weight") and P[k].ndim == 2 or k in ("wte", "wpe"):
            P[k] *= 10.0
    idx, tgt = S.uniform_tokens(2, 8, 64, seed=11)
    tgt[0, :3] = -1
    _fd_check(s, P, idx, tgt, None, np.random.default_rng(0))


def test_finite_differences_tiny_sampled():
    P = _params(TINY, seed=12, kind="random")
    idx, tgt = S.uniform_tokens(2, 24, 1024, seed=13)
    tgt[1, :10] = -1
    _fd_check(TINY, P, idx, tgt, 6, np.random.default_rng(1))


# ----------------------------------------------------------------------------
# Independent model from torch library layers, autograd and torch's optimiser.
# ----------------------------------------------------------------------------
def _torch_model(s, flat):
    """The pages' model written with torch library calls in float64 ("GPT-2
    from Scratch": CausalSelfAttention, MLP, Block, GPT.forward with the tied
    lm_head and F.cross_entropy(ignore_index=-1)). Returns (params, model)."""
    torch = pytest.importorskip("torch")
    F = torch.nn.functional
    names = [n for n, _ in O.layout(s)]
    shapes = dict(O.layout(s))
    P = {}
    off = 0
    for n in names:
        k = int(np.prod(shapes[n]))
        P[n] = torch.tensor(flat[off:off + k].reshape(shapes[n]), dtype=torch.float64, requires_grad=True)
        off += k
    C, H = s.n_embd, s.n_head

    def model(idx, tgt):
        idx_t = torch.tensor(idx, dtype=torch.long)
        tgt_t = torch.tensor(tgt, dtype=torch.long)
        B, T = idx_t.shape
        x = F.embedding(idx_t, P["wte"]) + F.embedding(torch.arange(T), P["wpe"])
        for l in range(s.n_layer):
            p = f"h.{l}."
            a = F.layer_norm(x, (C,), P[p + "ln_1.weight"], P[p + "ln_1.bias"], eps=1e-5)
            q, k, v = F.linear(a, P[p + "attn.c_attn.weight"], P[p + "attn.c_attn.bias"]).split(C, dim=2)
            q, k, v = (z.view(B, T, H, C // H).transpose(1, 2) for z in (q, k, v))
            y = F.scaled_dot_product_attention(q, k, v, is_causal=True)
            y = y.transpose(1, 2).contiguous().view(B, T, C)
            x = x + F.linear(y, P[p + "attn.c_proj.weight"], P[p + "attn.c_proj.bias"])
            m = F.layer_norm(x, (C,), P[p + "ln_2.weight"], P[p + "ln_2.bias"], eps=1e-5)
            u = F.gelu(F.linear(m, P[p + "mlp.c_fc.weight"], P[p + "mlp.c_fc.bias"]), approximate="tanh")
            x = x + F.linear(u, P[p + "mlp.c_proj.weight"], P[p + "mlp.c_proj.bias"])
        f = F.layer_norm(x, (C,), P["ln_f.weight"], P["ln_f.bias"], eps=1e-5)
        logits = F.linear(f, P["wte"])
        return F.cross_entropy(logits.view(-1, logits.size(-1)), tgt_t.view(-1), ignore_index=-1)

    return P, model


def _torch_model_step(s, flat, idx, tgt, lr, steps, max_norm=1.0):
    torch = pytest.importorskip("torch")
    P, model = _torch_model(s, flat)
    names = list(P)
    decay = [P[n] for n in names if P[n].dim() >= 2]
    nodecay = [P[n] for n in names if P[n].dim() < 2]
    opt = torch.optim.AdamW([{"params": decay, "weight_decay": 0.1},
                             {"params": nodecay, "weight_decay": 0.0}],
                            lr=lr, betas=(0.9, 0.95), eps=1e-8, foreach=False)
    out = []
    for _ in range(steps):
        opt.zero_grad(set_to_none=True)
        loss = model(idx, tgt)
        loss.backward()
        grads = {n: P[n].grad.detach().clone().numpy() for n in names}
        norm = torch.nn.utils.clip_grad_norm_(list(P.values()), max_norm)
        opt.step()
        out.append((loss.item(), float(norm), grads))
    params = {n: P[n].detach().numpy().copy() for n in names}
    return out, params


@pytest.mark.parametrize("max_norm", [1.0, 0.01])
def test_oracle_matches_torch_library_model(max_norm):
    s = TINY
    flat = S.random_params(S.ModelShape(2, 4, 128, 1024, 64), seed=14).astype(np.float64)
    idx, tgt = S.uniform_tokens(3, 33, 1024, seed=15)
    tgt[2, :9] = -1
    ref, ref_params = _torch_model_step(s, flat, idx, tgt, lr=6e-4, steps=2, max_norm=max_norm)
    P = O.unflatten(s, flat)
    M, V = O.zeros_like(s), O.zeros_like(s)
    for t in (1, 2):
        loss, norm, G = O.train_step(s, P, M, V, t, idx, tgt, lr=6e-4, max_norm=max_norm)
        rl, rn, rg = ref[t - 1]
        assert abs(loss - rl) < 1e-12
        assert abs(norm - rn) < 1e-12
        for n in G:
            assert np.max(np.abs(G[n] - rg[n])) < 1e-12 * max(1.0, np.max(np.abs(rg[n]))), n
    for n in P:
        assert np.max(np.abs(P[n] - ref_params[n])) < 1e-12, n


# ----------------------------------------------------------------------------
# Update closed forms ("Gradient clipping"; AdamW step 1).
# ----------------------------------------------------------------------------
def test_adamw_step1_closed_form_and_clip():
    s = MICRO
    rng = np.random.default_rng(16)
    P = _params(s, seed=17, kind="random")
    P0 = {k: v.copy() for k, v in P.items()}
    G = {k: rng.normal(size=v.shape) for k, v in P.items()}
    M, V = O.zeros_like(s), O.zeros_like(s)
    lr = 1e-3
    norm = O.adamw_update(s, P, G, M, V, 1, lr)
    true_norm = math.sqrt(sum((g * g).sum() for g in G.values()))
    assert abs(norm - true_norm) < 1e-12
    c = 1.0 / (true_norm + 1e-6)
    assert c < 1
    # post-clip norm = norm / (norm + 1e-6)
    post = math.sqrt(sum(((c * g) ** 2).sum() for g in G.values()))
    assert abs(post - true_norm / (true_norm + 1e-6)) < 1e-12
    for name, shp in O.layout(s):
        wd = 0.1 if len(shp) == 2 else 0.0
        cg = c * G[name]
        assert np.allclose(M[name], 0.1 * cg, rtol=1e-14, atol=0)
        assert np.allclose(V[name], 0.05 * cg * cg, rtol=1e-14, atol=0)
        expect = P0[name] * (1 - lr * wd) - lr * cg / (np.abs(cg) + 1e-8)
        assert np.allclose(P[name], expect, rtol=1e-12, atol=1e-16), name


def test_no_clip_below_threshold():
    s = MICRO
    P = _params(s, seed=18, kind="random")
    G = {k: np.full(v.shape, 1e-4) for k, v in P.items()}
    M, V = O.zeros_like(s), O.zeros_like(s)
    O.adamw_update(s, P, G, M, V, 1, 1e-3)
    assert np.allclose(M["wte"], 0.1 * 1e-4, rtol=1e-14)


def test_decay_groups():
    d = O.decays(TINY)
    assert d["wte"] == 0.1 and d["wpe"] == 0.1 and d["h.0.attn.c_attn.weight"] == 0.1
    assert d["h.1.mlp.c_proj.bias"] == 0.0 and d["h.0.ln_1.weight"] == 0.0 and d["ln_f.bias"] == 0.0


# ----------------------------------------------------------------------------
# Gradient accumulation ("Gradient accumulation, and the bug in getting it right").
# ----------------------------------------------------------------------------
def test_accumulation_equals_big_batch():
    s = TINY
    P = _params(s, seed=19, kind="random")
    idx, tgt = S.uniform_tokens(4, 20, 1024, seed=20)
    loss_big, _, cache = O.forward(s, P, idx, tgt)
    G_big = O.backward(s, P, cache)
    loss_acc, G_acc = O.accumulate_grads(s, P, [(idx[i:i + 1], tgt[i:i + 1]) for i in range(4)])
    assert abs(loss_big - loss_acc) < 1e-12
    for n in G_big:
        assert np.max(np.abs(G_big[n] - G_acc[n])) < 1e-13, n


def _masked_micro_batches():
    """Four micro-batches whose targets carry masked prefixes of different
    lengths (the supervised fine-tuning masking of "Pretraining and
    fine-tuning nanoGPT-124M from scratch"), so every micro-batch has its own
    count of valid targets; the last one is fully valid."""
    batches = []
    for k, n_masked in enumerate([3, 11, 0, 17]):
        idx, tgt = S.uniform_tokens(2, 24, 1024, seed=40 + k)
        tgt[0, :n_masked] = -1
        tgt[1, :n_masked // 2] = -1
        batches.append((idx, tgt))
    return batches


def _torch_accumulation(s, flat, batches):
    """The pages' accumulation loop with library calls ("Gradient
    accumulation, and the bug in getting it right"): each micro-batch's
    F.cross_entropy(ignore_index=-1) divided by the number of micro-batches,
    backward() adding into .grad; the reported loss is the sum of the scaled
    micro losses."""
    P, model = _torch_model(s, flat)
    total = 0.0
    for idx, tgt in batches:
        loss = model(idx, tgt) / len(batches)
        loss.backward()
        total += loss.item()
    return total, {n: P[n].grad.detach().numpy().copy() for n in P}


def _max_grad_err(G, ref):
    return max(np.max(np.abs(G[n] - ref[n])) / max(1.0, np.max(np.abs(ref[n]))) for n in ref)


def test_accumulation_with_masks_matches_torch_loop():
    s = TINY
    flat = S.random_params(_syn(s), seed=41).astype(np.float64)
    batches = _masked_micro_batches()
    assert len({int((t != -1).sum()) for _, t in batches}) == 4   # valid counts all differ
    ref_loss, ref_G = _torch_accumulation(s, flat, batches)
    loss, G = O.accumulate_grads(s, O.unflatten(s, flat), batches)
    assert abs(loss - ref_loss) < 1e-12
    assert _max_grad_err(G, ref_G) < 1e-12


def test_accumulation_token_weighted_mean_is_rejected():
    """Planted mistake: a token-weighted global mean over all micro-batches
    (each micro-batch weighted by its share of the valid targets) instead of
    the per-micro-batch mean divided by the number of micro-batches. With
    unequal valid counts the two differ, and the torch loop tells them apart."""
    s = TINY
    flat = S.random_params(_syn(s), seed=41).astype(np.float64)
    batches = _masked_micro_batches()
    ref_loss, ref_G = _torch_accumulation(s, flat, batches)
    P = O.unflatten(s, flat)
    n_valid = [int((t != -1).sum()) for _, t in batches]
    G = O.zeros_like(s)
    loss = 0.0
    for (idx, tgt), nv in zip(batches, n_valid):
        l_k, _, cache = O.forward(s, P, idx, tgt)
        w = nv / sum(n_valid)
        g = O.backward(s, P, cache, loss_scale=w)
        for k in G:
            G[k] += g[k]
        loss += w * l_k
    assert abs(loss - ref_loss) > 1e-4
    assert _max_grad_err(G, ref_G) > 1e-6


# ----------------------------------------------------------------------------
# Weight tying: one wte row feeds both the input and its logit column.
# ----------------------------------------------------------------------------
def test_tying_changes_input_and_output():
    s = TINY
    P = _params(s, seed=21, kind="random")
    idx = np.array([[5, 6, 7]])
    _, la, _ = O.forward(s, P, idx)
    rng = np.random.default_rng(0)           # random vectors: LayerNorm removes constant shifts
    P["wte"][900] += rng.normal(size=128)    # a token that is not in the input
    _, lb, _ = O.forward(s, P, idx)
    d = np.abs(la - lb)[0]
    assert d[:, 900].min() > 0 and np.array_equal(np.delete(d, 900, axis=1), np.zeros((3, 1023)))
    P["wte"][6] += rng.normal(size=128)   # the token at position 1: positions >= 1 move everywhere,
    _, lc, _ = O.forward(s, P, idx)     # position 0 only in its output column 6
    d0 = np.abs(lb[0, 0] - lc[0, 0])
    assert d0[6] > 0 and np.array_equal(np.delete(d0, 6), np.zeros(1023))
    assert np.abs(lb[0, 1:] - lc[0, 1:]).min() > 0


# ----------------------------------------------------------------------------
# Overfitting one batch ("Debugging checklist" item 4).
# ----------------------------------------------------------------------------
@pytest.mark.slow
def test_overfit_single_batch():
    s = O.Shape(n_layer=2, n_head=4, n_embd=64, vocab_size=128, block_size=16)
    P = O.unflatten(s, S.init_params(S.ModelShape(2, 4, 64, 128, 16), seed=22))
    M, V = O.zeros_like(s), O.zeros_like(s)
    idx, tgt = S.uniform_tokens(2, 16, 128, seed=23)
    first = None
    for t in range(1, 201):
        loss, _, _ = O.train_step(s, P, M, V, t, idx, tgt, lr=3e-3)
        first = first if first is not None else loss
    assert first > 4.5 and loss < 0.1, (first, loss)


# ----------------------------------------------------------------------------
# The pins are sensitive: a planted mistake in the oracle's backward fails them.
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("mutation", ["ln_drop_term", "gelu_grad_const", "attn_rowsum", "tie_scatter",
                                      "scatter_drops_repeats"])
def test_planted_mistakes_are_caught(monkeypatch, mutation):
    if mutation == "ln_drop_term":
        def bad(dy, saved, w):
            xhat, rstd = saved
            dxhat = dy * w
            dx = rstd * (dxhat - dxhat.mean(axis=-1, keepdims=True))
            return dx, (dy * xhat).reshape(-1, dy.shape[-1]).sum(0), dy.reshape(-1, dy.shape[-1]).sum(0)
        monkeypatch.setattr(O, "layer_norm_backward", bad)
    elif mutation == "gelu_grad_const":
        good = O.gelu_tanh_grad
        monkeypatch.setattr(O, "gelu_tanh_grad", lambda u: good(u) * 1.01)
    elif mutation == "attn_rowsum":
        def bad(dy, q, k, v, p):
            hd = q.shape[-1]
            dv = np.swapaxes(p, -1, -2) @ dy
            ds = p * (dy @ np.swapaxes(v, -1, -2))
            return (ds @ k) / math.sqrt(hd), (np.swapaxes(ds, -1, -2) @ q) / math.sqrt(hd), dv
        monkeypatch.setattr(O, "causal_attention_backward", bad)
    elif mutation == "tie_scatter":
        good_backward = O.backward

        def bad_backward(s, P, cache, loss_scale=1.0):
            G = good_backward(s, P, cache, loss_scale)
            G["wte"][cache["idx"].reshape(-1)] *= 0.5      # lose part of the embedding scatter
            return G
        monkeypatch.setattr(O, "backward", bad_backward)
    elif mutation == "scatter_drops_repeats":
        def bad(idx, dx, V, block_size):
            C = dx.shape[-1]
            dwte = np.zeros((V, C))
            dwte[idx.reshape(-1)] += dx.reshape(-1, C)   # buffered: a repeated id keeps one row
            dwpe = np.zeros((block_size, C))
            dwpe[:idx.shape[1]] = dx.sum(axis=0)
            return dwte, dwpe
        monkeypatch.setattr(O, "embedding_backward", bad)
    s = MICRO
    P = _params(s, seed=30, kind="random")
    for k in P:
        if P[k].ndim == 2:
            P[k] *= 10.0
    idx, tgt = S.uniform_tokens(2, 8, 64, seed=31)   # ids 43 and 11 occur twice
    coords = None if mutation == "scatter_drops_repeats" else 8   # every coordinate reaches the repeated rows
    with pytest.raises(AssertionError):
        _fd_check(s, P, idx, tgt, coords, np.random.default_rng(2))


# ----------------------------------------------------------------------------
# Learning-rate schedule ("GPT-2 from Scratch", "Warmup and cosine decay")
# ----------------------------------------------------------------------------
def test_lr_schedule_page_properties():
    """The page fixes: a linear ramp from zero over the warmup, the peak at
    t = t_w (cos 0 = 1), the floor at t = t_max (cos pi = -1), the midpoint
    halfway, and a floor of 10% of the peak; the 124M run's numbers."""
    g = GOLDEN["lr_schedule"]
    r = GOLDEN["lr_schedule_124m_run"]
    mx, mn, tw, tm = r["max_lr"], r["min_lr"], r["warmup_steps"], r["max_steps"]
    assert mx == g["max_lr"] and mn == g["min_lr"] and abs(mn - 0.1 * mx) < 1e-18
    lr = lambda k: O.lr_schedule(k, mx, mn, tw, tm)   # noqa: E731
    assert lr(0) == pytest.approx(mx / tw)              # first step of the ramp
    assert lr(tw - 1) == pytest.approx(mx)              # end of the ramp
    ramp = [lr(k) for k in range(tw)]
    assert all(b - a == pytest.approx(mx / tw) for a, b in zip(ramp, ramp[1:]))   # linear
    assert lr(tw) == pytest.approx(mx)                  # cos 0 = 1
    assert lr(tm) == pytest.approx(mn)                  # cos pi = -1
    assert lr((tw + tm) / 2) == pytest.approx((mx + mn) / 2)
    assert lr(tm + 1) == mn and lr(10 * tm) == mn
    decay = [lr(k) for k in range(tw, tm + 1, 97)]
    assert all(b <= a for a, b in zip(decay, decay[1:]))


def test_lr_schedule_planted_mistakes_are_caught():
    """A schedule that forgets the +1 of the ramp, or decays with the full
    cosine period, or floors at zero, breaks one of the page's properties."""
    mx, mn, tw, tm = 6e-4, 6e-5, 10, 110
    wrong_ramp = lambda k: mx * k / tw if k < tw else O.lr_schedule(k, mx, mn, tw, tm)   # noqa: E731
    assert wrong_ramp(tw - 1) != pytest.approx(mx)
    wrong_period = lambda k: mn + (mx - mn) * 0.5 * (1 + np.cos(2 * np.pi * (k - tw) / (tm - tw)))   # noqa: E731
    assert wrong_period(tm) != pytest.approx(O.lr_schedule(tm, mx, mn, tw, tm))
    assert O.lr_schedule(tm, mx, 0.0, tw, tm) != pytest.approx(mn)


# ----------------------------------------------------------------------------
# Sampling and generation ("GPT-2 from Scratch", "A generation loop").
# ----------------------------------------------------------------------------
def _torch_topk_softmax(logits, temperature, top_k):
    torch = pytest.importorskip("torch")
    x = torch.tensor(logits, dtype=torch.float64) / temperature
    if top_k >= 1:
        v, _ = torch.topk(x, min(top_k, x.numel()))
        x = torch.where(x < v[-1], torch.tensor(float("-inf"), dtype=torch.float64), x)
    return torch.softmax(x, dim=-1).numpy()


@pytest.mark.parametrize("temperature,top_k", [(1.0, 0), (0.7, 5), (1.6, 12), (0.8, 40)])
def test_sample_frequencies_match_torch_softmax(temperature, top_k):
    """Over a uniform grid of u, each index is drawn with the probability torch's
    softmax of the temperature-scaled, top-k-masked row gives it: this fixes the
    temperature (divide), the mask (drop below the k-th, keep the rest) and the
    order of the inverse CDF (inclusive, vocabulary order)."""
    rng = np.random.default_rng(31)
    logits = rng.normal(0.0, 1.5, 48)
    n = 20_000
    us = (np.arange(n) + 0.5) / n
    counts = np.zeros(48)
    draws = []
    for u in us:
        j, probs, _ = O.sample_next(logits, temperature, top_k, u)
        counts[j] += 1
        draws.append(j)
    ref = _torch_topk_softmax(logits, temperature, top_k)
    assert np.max(np.abs(counts / n - ref)) <= 1.0 / n + 1e-12
    assert np.max(np.abs(probs - ref)) < 1e-12
    # inverse CDF in vocabulary order: the draw never decreases as u grows
    assert all(a <= b for a, b in zip(draws, draws[1:]))


def test_sample_top1_is_argmax_and_ties_at_kth_stay():
    rng = np.random.default_rng(32)
    x = rng.normal(size=100)
    for u in (0.0, 0.3, 0.999999):
        assert O.sample_next(x, 0.9, 1, u)[0] == int(np.argmax(x))
    # three entries equal to the 2nd largest value all stay with top_k = 2
    x = np.array([0.0, 4.0, 1.0, 4.0, 5.0, 4.0, -1.0])
    _, probs, _ = O.sample_next(x, 1.0, 2, 0.5)
    kept = np.nonzero(probs > 0)[0].tolist()
    assert kept == [1, 3, 4, 5]
    e = np.exp(np.array([4.0, 4.0, 5.0, 4.0]) - 5.0)
    assert np.allclose(probs[kept], e / e.sum(), rtol=1e-14)
    # top_k >= V and top_k <= 0 keep everything
    for k in (0, -3, 7, 50):
        assert np.all(O.sample_next(x, 1.0, k, 0.5)[1] > 0)


def test_sample_margin_and_last_index():
    x = np.log(np.array([0.25, 0.25, 0.5]))
    j, probs, margin = O.sample_next(x, 1.0, 0, 0.3)
    assert j == 1 and abs(margin - 0.05) < 1e-12          # interval [0.25, 0.5)
    assert O.sample_next(x, 1.0, 0, 0.5)[0] == 2          # u on a boundary: the next index
    assert O.sample_next(x, 1.0, 0, 0.0)[0] == 0
    # with top-k the masked tail is never drawn, even at u -> 1
    assert O.sample_next(np.array([3.0, 2.0, 1.0, 0.0]), 1.0, 2, 1.0 - 1e-15)[0] == 1


def _torch_last_logits(s, flat, idx):
    torch = pytest.importorskip("torch")
    F = torch.nn.functional
    P, off = {}, 0
    for n, shp in O.layout(s):
        k = int(np.prod(shp))
        P[n] = torch.tensor(flat[off:off + k].reshape(shp), dtype=torch.float64)
        off += k
    C, H = s.n_embd, s.n_head
    x_idx = torch.tensor(idx, dtype=torch.long)
    B, T = x_idx.shape
    x = F.embedding(x_idx, P["wte"]) + F.embedding(torch.arange(T), P["wpe"])
    for l in range(s.n_layer):
        p = f"h.{l}."
        a = F.layer_norm(x, (C,), P[p + "ln_1.weight"], P[p + "ln_1.bias"], eps=1e-5)
        q, k, v = F.linear(a, P[p + "attn.c_attn.weight"], P[p + "attn.c_attn.bias"]).split(C, dim=2)
        q, k, v = (z.view(B, T, H, C // H).transpose(1, 2) for z in (q, k, v))
        y = F.scaled_dot_product_attention(q, k, v, is_causal=True).transpose(1, 2).reshape(B, T, C)
        x = x + F.linear(y, P[p + "attn.c_proj.weight"], P[p + "attn.c_proj.bias"])
        m = F.layer_norm(x, (C,), P[p + "ln_2.weight"], P[p + "ln_2.bias"], eps=1e-5)
        u = F.gelu(F.linear(m, P[p + "mlp.c_fc.weight"], P[p + "mlp.c_fc.bias"]), approximate="tanh")
        x = x + F.linear(u, P[p + "mlp.c_proj.weight"], P[p + "mlp.c_proj.bias"])
    f = F.layer_norm(x, (C,), P["ln_f.weight"], P["ln_f.bias"], eps=1e-5)
    return F.linear(f[:, -1, :], P["wte"]).numpy()


def test_generate_top1_matches_greedy_torch_model_past_block_size():
    """top_k = 1 makes every draw the argmax: the oracle's loop must then equal
    greedy decoding with torch's library layers, including the crop to the
    last block_size tokens once the sequence outgrows the block."""
    s = MICRO
    flat = S.random_params(_syn(s), seed=33).astype(np.float64)
    P = O.unflatten(s, flat)
    idx, _ = S.uniform_tokens(2, 5, s.vocab_size, seed=34)
    n_new = 7                                   # 5 + 7 > block_size = 8
    u = np.random.default_rng(35).random((n_new, 2))
    seq, margins = O.generate(s, P, idx, n_new, 0.9, 1, u)
    ref = np.asarray(idx).copy()
    for _ in range(n_new):
        lg = _torch_last_logits(s, flat, ref[:, -s.block_size:])
        ref = np.concatenate([ref, lg.argmax(axis=-1)[:, None]], axis=1)
    assert seq.shape == (2, 12)
    assert np.array_equal(seq, ref)
    assert np.all(margins >= 0)


def test_generate_draws_follow_torch_probabilities():
    """One draw of the loop at a given u is the inverse CDF of torch's softmax of
    the last-position logits of the torch model (temperature and top-k applied)."""
    s = MICRO
    flat = S.random_params(_syn(s), seed=36).astype(np.float64)
    P = O.unflatten(s, flat)
    idx, _ = S.uniform_tokens(3, 6, s.vocab_size, seed=37)
    u = np.random.default_rng(38).random((1, 3))
    seq, _ = O.generate(s, P, idx, 1, 0.8, 10, u)
    lg = _torch_last_logits(s, flat, idx)
    for b in range(3):
        cdf = np.cumsum(_torch_topk_softmax(lg[b], 0.8, 10))
        assert seq[b, -1] == int(np.searchsorted(cdf, u[0, b], side="right"))


def test_sample_low_temperature_limit_and_empty_generation():
    """As the temperature goes to 0 the softmax concentrates on the maximum, so
    every u away from 0 and 1 draws the argmax; a generation of no new tokens
    returns the prompt unchanged."""
    x = np.array([0.3, 1.2, -0.5, 1.1, 0.0])
    for u in (1e-6, 0.25, 0.5, 0.999):
        j, probs, _ = O.sample_next(x, 1e-3, 0, u)
        assert j == 1 and probs[1] > 1.0 - 1e-12
    s = MICRO
    P = _params(s, seed=3)
    idx, _ = S.uniform_tokens(2, 4, s.vocab_size, seed=39)
    seq, margins = O.generate(s, P, idx, 0, 1.0, 0, np.zeros((0, 2)))
    assert np.array_equal(seq, idx) and margins.shape == (0, 2)
