"""Parity of the CUDA path (through the C ABI) with the float64 CPU oracle.

Tolerances (metric: per tensor max|gpu - oracle| / max|oracle|):
  fp32 mode: loss 1e-5 relative, logits and gradients 1e-4, parameters after
             AdamW 1e-5 absolute (elements whose oracle gradient is below ten
             times the tensor's observed gradient error are reported and
             excluded: AdamW's first step moves them by ~lr * sign(g), so the
             sign of a gradient inside the error band decides a 1.2e-3 move).
  bf16 mode: loss 2e-2 absolute, per-tensor gradient cosine >= 0.999.
"""
import math

import numpy as np
import pytest

from oracle import gpt2_oracle as O
from decoder_only_transformer_sm_b200 import synthetic as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TINY = S.TINY


def _oshape(s):
    return O.Shape(s.n_layer, s.n_head, s.n_embd, s.vocab_size, s.block_size)


def _model(s, precision, B, T, seed=0, grad_clip=1.0):
    from decoder_only_transformer_sm_b200 import native
    return native.GPT2(s.n_layer, s.n_head, s.n_embd, s.vocab_size, s.block_size, B, T,
                       precision=precision, seed=seed, grad_clip=grad_clip)


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(float(np.max(np.abs(b))), 1e-30))


def _cos(a, b):
    a = a.astype(np.float64).ravel()
    b = b.astype(np.float64).ravel()
    na, nb = np.linalg.norm(a), np.linalg.norm(b)
    if na == 0 and nb == 0:
        return 1.0
    return float(a @ b / (na * nb))


def _split(s, flat):
    return O.unflatten(_oshape(s), flat)


def _check_params_fp32(s, p_gpu, p_ref, g_gpu, g_ref, tol=1e-5):
    """Post-AdamW params within tol, excluding the sign-hazard elements."""
    Pg, Pr, Gg, Gr = _split(s, p_gpu), _split(s, p_ref), _split(s, g_gpu), _split(s, g_ref)
    excluded = 0
    for name in Pr:
        gerr = np.max(np.abs(Gg[name] - Gr[name]))
        ok = np.abs(Gr[name]) >= 10 * gerr
        excluded += int((~ok).sum())
        d = np.abs(Pg[name] - Pr[name])[ok]
        assert d.size == 0 or d.max() <= tol, (name, float(d.max()))
    return excluded


# ----------------------------------------------------------------------------
# fp32 mode, tiny config (2 layers, C = 128, V = 1024): the small parity case.
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("kind", ["init", "random"])
def test_tiny_fp32_step_matches_oracle(kind):
    s = TINY
    B, T = 4, 64
    flat = S.init_params(s, seed=0) if kind == "init" else S.random_params(s, seed=5)
    idx, tgt = S.uniform_tokens(B, T, s.vocab_size, seed=1000)
    m = _model(s, "fp32", B, T)
    m.set_params(flat)
    di, dt = _dev(idx), _dev(tgt)
    logits = torch.empty((B, T, s.vocab_size), dtype=torch.float32, device="cuda")
    loss_f = m.forward(di, dt, logits)
    # oracle
    P = O.unflatten(_oshape(s), flat.astype(np.float64))
    ref_loss, ref_logits, _ = O.forward(_oshape(s), P, idx, tgt)
    assert abs(loss_f - ref_loss) / ref_loss < 1e-5
    assert _rel(logits.cpu().numpy(), ref_logits) < 1e-4
    M, V = O.zeros_like(_oshape(s)), O.zeros_like(_oshape(s))
    ref_loss2, ref_norm, G = O.train_step(_oshape(s), P, M, V, 1, idx, tgt, lr=6e-4)
    loss, norm = m.step(di, dt, 6e-4)
    assert abs(loss - ref_loss2) / ref_loss2 < 1e-5
    assert abs(norm - ref_norm) / ref_norm < 1e-4
    g = m.get_grads()
    Gg = _split(s, g)
    for name in G:
        assert _rel(Gg[name], G[name]) < 1e-4, (name, _rel(Gg[name], G[name]))
    excluded = _check_params_fp32(s, m.get_params(), O.flatten(_oshape(s), P), g, O.flatten(_oshape(s), G))
    assert excluded < 0.01 * m.n_params, excluded
    mm, vv, t = m.get_opt_state()
    assert t == 1
    assert _rel(mm, O.flatten(_oshape(s), M)) < 1e-4
    assert _rel(vv, O.flatten(_oshape(s), V)) < 1e-4
    m.close()


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
@pytest.mark.parametrize("C,H", [(768, 12), (1024, 16), (1280, 20), (1600, 25)])
def test_gpt2_width_one_layer_grads(precision, C, H):
    """The widths of GPT-2 small, medium, large and XL (head width 64; C = 1600
    is not a multiple of 128, so the row kernels' last lane group is partial),
    one layer each with a small vocabulary and ragged T."""
    s = S.ModelShape(n_layer=1, n_head=H, n_embd=C, vocab_size=512, block_size=64)
    B, T = 3, 37
    idx, tgt = S.uniform_tokens(B, T, s.vocab_size, seed=77)
    tgt[1, :5] = -1
    flat = S.random_params(s, seed=78)
    P = O.unflatten(_oshape(s), flat.astype(np.float64))
    Mo, Vo = O.zeros_like(_oshape(s)), O.zeros_like(_oshape(s))
    ref_loss, ref_norm, G = O.train_step(_oshape(s), P, Mo, Vo, 1, idx, tgt, lr=1e-4)
    m = _model(s, precision, B, T)
    m.set_params(flat)
    loss, norm = m.step(_dev(idx), _dev(tgt), 1e-4)
    Gg = _split(s, m.get_grads())
    if precision == "fp32":
        assert abs(loss - ref_loss) / ref_loss < 1e-5
        assert abs(norm - ref_norm) / ref_norm < 1e-4
        for name in G:
            assert _rel(Gg[name], G[name]) < 1e-4, (name, _rel(Gg[name], G[name]))
    else:
        assert abs(loss - ref_loss) < 2e-2
        for name in G:
            assert _cos(Gg[name], G[name]) >= 0.999, name
            nr, ng = np.linalg.norm(G[name]), np.linalg.norm(Gg[name].astype(np.float64))
            assert nr == 0 or abs(ng / nr - 1.0) < 1e-2, (name, ng, nr)
    m.close()


def test_tiny_fp32_three_steps_and_ragged_shape():
    """B=3, T=37: partial attention tiles and GEMM edges; AdamW steps 1..3.

    Each step starts both sides from the oracle's state (parameters, moments,
    step count), so every step is held to the single-step tolerances: without
    the re-sync, the sign-hazard elements of step 1 (moved by ~2 lr) change
    the gradients of later steps by more than 1e-4."""
    s = TINY
    B, T = 3, 37
    flat = S.random_params(s, seed=7)
    idx, tgt = S.uniform_tokens(B, T, s.vocab_size, seed=8)
    tgt[1, :11] = -1
    m = _model(s, "fp32", 4, 64)
    P = O.unflatten(_oshape(s), flat.astype(np.float64))
    M, V = O.zeros_like(_oshape(s)), O.zeros_like(_oshape(s))
    di, dt = _dev(idx), _dev(tgt)
    for t in (1, 2, 3):
        m.set_params(O.flatten(_oshape(s), P).astype(np.float32))
        m.set_opt_state(O.flatten(_oshape(s), M), O.flatten(_oshape(s), V), t - 1)
        ref_loss, ref_norm, G = O.train_step(_oshape(s), P, M, V, t, idx, tgt, lr=1e-3)
        loss, norm = m.step(di, dt, 1e-3)
        assert abs(loss - ref_loss) / ref_loss < 1e-5, t
        assert abs(norm - ref_norm) / ref_norm < 1e-4, t
        g = m.get_grads()
        for name, ref in G.items():
            assert _rel(_split(s, g)[name], ref) < 1e-4, (t, name)
        _check_params_fp32(s, m.get_params(), O.flatten(_oshape(s), P), g, O.flatten(_oshape(s), G))
        mm, vv, tt = m.get_opt_state()
        assert tt == t
    m.close()


def test_tiny_fp32_accumulation_with_masks():
    s = TINY
    flat = S.random_params(s, seed=9)
    batches = S.accumulation_batches(4, 2, 64, s.vocab_size, seed=10)
    m = _model(s, "fp32", 2, 64)
    m.set_params(flat)
    m.zero_grad()
    for idx, tgt in batches:
        m.accumulate(_dev(idx), _dev(tgt), 1.0 / len(batches))
    loss, norm = m.update(6e-4)
    P = O.unflatten(_oshape(s), flat.astype(np.float64))
    ref_loss, G = O.accumulate_grads(_oshape(s), P, batches)
    assert abs(loss - ref_loss) / ref_loss < 1e-5
    assert abs(norm - O.grad_norm(G)) / O.grad_norm(G) < 1e-4
    g = m.get_grads()
    for name, ref in G.items():
        assert _rel(_split(s, g)[name], ref) < 1e-4, name
    m.close()


def test_tiny_fp32_forced_clip_and_T1():
    s = TINY
    flat = S.random_params(s, seed=11)
    idx, tgt = S.uniform_tokens(2, 1, s.vocab_size, seed=12)
    m = _model(s, "fp32", 2, 64, grad_clip=0.01)
    m.set_params(flat)
    loss, norm = m.step(_dev(idx), _dev(tgt), 6e-4)
    P = O.unflatten(_oshape(s), flat.astype(np.float64))
    M, V = O.zeros_like(_oshape(s)), O.zeros_like(_oshape(s))
    ref_loss, ref_norm, G = O.train_step(_oshape(s), P, M, V, 1, idx, tgt, lr=6e-4, max_norm=0.01)
    assert ref_norm > 0.01
    assert abs(loss - ref_loss) / ref_loss < 1e-5 and abs(norm - ref_norm) / ref_norm < 1e-4
    _check_params_fp32(s, m.get_params(), O.flatten(_oshape(s), P), m.get_grads(), O.flatten(_oshape(s), G))
    m.close()


def test_all_targets_ignored_gives_zero_loss_and_grads():
    s = TINY
    idx, _ = S.uniform_tokens(2, 16, s.vocab_size, seed=13)
    tgt = np.full((2, 16), -1, np.int32)
    m = _model(s, "fp32", 2, 16)
    loss, norm = m.step(_dev(idx), _dev(tgt), 6e-4)
    assert loss == 0.0 and norm == 0.0
    assert not m.get_grads().any()
    m.close()


def test_causal_invariance_on_gpu():
    s = TINY
    idx, _ = S.uniform_tokens(2, 40, s.vocab_size, seed=14)
    idx2 = idx.copy()
    idx2[:, 18:] = (idx2[:, 18:] + 77) % s.vocab_size
    m = _model(s, "fp32", 2, 40)
    m.set_params(S.random_params(s, seed=15))
    la = torch.empty((2, 40, s.vocab_size), device="cuda")
    lb = torch.empty_like(la)
    m.forward(_dev(idx), None, la)
    m.forward(_dev(idx2), None, lb)
    assert torch.equal(la[:, :18], lb[:, :18])
    assert not torch.allclose(la[:, 18:], lb[:, 18:])
    m.close()


def _state(m):
    mm, vv, t = m.get_opt_state()
    return m.get_params(), mm, vv, t


def _assert_same_state(a, b):
    """Bit-identical parameters, moments and step counter (NaNs included)."""
    for x, y in zip(a[:3], b[:3]):
        assert x.tobytes() == y.tobytes()
    assert a[3] == b[3]


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_bad_token_leaves_state_unchanged(precision):
    """A step that reports BAD_TOKEN (an id outside [0, V) in the forward) must
    not move the weights, the moments or the step counter ("The loop": the
    update belongs to a valid step), and the report clears the flag: the next
    valid step succeeds and counts as step 2."""
    from decoder_only_transformer_sm_b200 import native
    s = TINY
    m = _model(s, precision, 2, 8)
    m.set_params(S.random_params(s, seed=16))
    idx, tgt = S.uniform_tokens(2, 8, s.vocab_size, seed=16)
    m.step(_dev(idx), _dev(tgt), 6e-4)                      # t = 1, moments non-zero
    before = _state(m)
    bad = idx.copy()
    bad[0, 3] = s.vocab_size + 5
    for _ in range(3):                                      # eager, graph capture, graph replay
        with pytest.raises(native.Gpt2Error) as e:
            m.step(_dev(bad), _dev(tgt), 6e-4)
        assert e.value.code == -6
        _assert_same_state(before, _state(m))
    badt = tgt.copy()
    badt[1, 0] = s.vocab_size
    with pytest.raises(native.Gpt2Error) as e:              # an out-of-range target
        m.step(_dev(idx), _dev(badt), 6e-4)
    assert e.value.code == -6
    _assert_same_state(before, _state(m))
    m.step(_dev(idx), _dev(tgt), 6e-4)
    assert _state(m)[3] == 2
    m.close()


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_nonfinite_step_leaves_state_unchanged(precision):
    """A NaN parameter (made on the host through gpt2_set_params) gives a
    non-finite loss and norm: the step returns NONFINITE and parameters,
    moments and the step counter stay bit-identical ("Gradient clipping" needs
    a finite norm)."""
    from decoder_only_transformer_sm_b200 import native
    s = TINY
    m = _model(s, precision, 2, 8)
    flat = S.random_params(s, seed=23)
    m.set_params(flat)
    idx, tgt = S.uniform_tokens(2, 8, s.vocab_size, seed=24)
    m.step(_dev(idx), _dev(tgt), 6e-4)
    p = m.get_params()
    p[12345] = np.nan                                       # inside wte: reaches the logits
    m.set_params(p)
    before = _state(m)
    with pytest.raises(native.Gpt2Error) as e:
        m.step(_dev(idx), _dev(tgt), 6e-4)
    assert e.value.code == -5
    _assert_same_state(before, _state(m))
    m.close()


def test_device_init_matches_recipe_and_initial_loss():
    s = TINY
    m = _model(s, "fp32", 4, 64, seed=123)
    P = _split(s, m.get_params())
    assert abs(P["wte"].std() - 0.02) < 1e-3 and abs(P["wte"].mean()) < 1e-3
    assert abs(P["h.1.mlp.c_proj.weight"].std() - 0.02 / math.sqrt(4)) < 1e-3
    assert np.all(P["h.0.ln_2.weight"] == 1) and not P["h.0.attn.c_attn.bias"].any()
    idx, tgt = S.uniform_tokens(4, 64, s.vocab_size, seed=1000)
    loss = m.forward(_dev(idx), _dev(tgt))
    assert abs(loss - (math.log(1024) + 0.5 * 0.02 ** 2 * 128)) < 0.05
    m.close()


# ----------------------------------------------------------------------------
# bf16 mode.
# ----------------------------------------------------------------------------
def _bf16_check(s, flat, idx, tgt, lr=6e-4):
    m = _model(s, "bf16", idx.shape[0], idx.shape[1])
    m.set_params(flat)
    loss, norm = m.step(_dev(idx), _dev(tgt), lr)
    g = m.get_grads()
    P = O.unflatten(_oshape(s), flat.astype(np.float64))
    M, V = O.zeros_like(_oshape(s)), O.zeros_like(_oshape(s))
    ref_loss, ref_norm, G = O.train_step(_oshape(s), P, M, V, 1, idx, tgt, lr=lr)
    assert abs(loss - ref_loss) < 2e-2, (loss, ref_loss)
    Gg = _split(s, g)
    worst = min((_cos(Gg[n], G[n]), n) for n in G)
    assert worst[0] >= 0.999, worst
    # cosine ignores scale: the norms must agree too (bf16 roundings are about
    # 2^-8 relative and largely cancel in a norm; 1e-2 leaves a wide margin)
    for n in G:
        nr, ng = np.linalg.norm(G[n]), np.linalg.norm(Gg[n].astype(np.float64))
        if nr > 0:
            assert abs(ng / nr - 1.0) < 1e-2, (n, ng, nr)
    m.close()
    return loss, ref_loss, worst


def test_tiny_bf16_step_matches_oracle():
    s = TINY
    idx, tgt = S.uniform_tokens(4, 64, s.vocab_size, seed=1000)
    _bf16_check(s, S.random_params(s, seed=17), idx, tgt)


def test_tiny_bf16_ragged():
    s = TINY
    idx, tgt = S.uniform_tokens(3, 45, s.vocab_size, seed=18)
    tgt[0, :20] = -1
    _bf16_check(s, S.random_params(s, seed=19), idx, tgt)


def test_bf16_accumulation_with_masks_matches_oracle():
    """Gradient accumulation in bf16 mode on the 124M width (one block, C=768,
    12 heads, head width 64, so the tensor-core GEMMs and attention run):
    zero_grad + 4 x accumulate(1/4) + update over the accumulation workload's
    micro-batches, the second half with masked target prefixes ("Gradient
    accumulation, and the bug in getting it right"; "Supervised fine-tuning").
    Against oracle.accumulate_grads + adamw_update: loss 2e-2 absolute,
    per-tensor gradient cosine >= 0.999, gradient norms within 1%, the global
    norm within 1%, and the post-update parameters within 2*lr of the oracle's
    (AdamW's first step moves each element by about lr)."""
    s = S.ModelShape(1, 12, 768, 1024, 128)
    os_ = _oshape(s)
    n_micro, B, T, lr = 4, 2, 128, 6e-4
    flat = S.random_params(s, seed=61)
    batches = S.accumulation_batches(n_micro, B, T, s.vocab_size, seed=62)
    assert all((t == -1).any() for _, t in batches[n_micro // 2:])
    m = _model(s, "bf16", B, T)
    m.set_params(flat)
    m.zero_grad()
    for idx, tgt in batches:
        m.accumulate(_dev(idx), _dev(tgt), 1.0 / n_micro)
    g = m.get_grads()
    loss, norm = m.update(lr)
    P = O.unflatten(os_, flat.astype(np.float64))
    ref_loss, G = O.accumulate_grads(os_, P, batches)
    ref_norm = O.grad_norm(G)
    assert abs(loss - ref_loss) < 2e-2, (loss, ref_loss)
    assert abs(norm / ref_norm - 1.0) < 1e-2, (norm, ref_norm)
    Gg = _split(s, g)
    worst = min((_cos(Gg[n], G[n]), n) for n in G)
    assert worst[0] >= 0.999, worst
    for n in G:
        nr, ng = np.linalg.norm(G[n]), np.linalg.norm(Gg[n].astype(np.float64))
        if nr > 0:
            assert abs(ng / nr - 1.0) < 1e-2, (n, ng, nr)
    M, V = O.zeros_like(os_), O.zeros_like(os_)
    O.adamw_update(os_, P, G, M, V, 1, lr)
    assert np.max(np.abs(m.get_params() - O.flatten(os_, P))) <= 2 * lr + 1e-6
    m.close()


def test_embedding_gradient_is_deterministic():
    """The token-embedding gradient adds each token's rows in row order (a sort by
    token, then sums of each token's run), not with atomics: in fp32 mode, whose
    other kernels have fixed summation orders too at this shape, two identical
    gradient passes give a bit-identical wte gradient. The shape keeps the tied
    lm_head's weight gradient, the other term of that gradient, off split-K (V x C
    has more 128 x 256 tiles than the GPU has SMs). Zipf tokens repeat many ids
    (the most frequent one thousands of times, across many windows of the sorted
    list), and 20480 rows are more than one sort tile (16384). (In bf16 mode the
    rows reaching the embedding already differ in their last bits from pass to
    pass: the attention backward adds dQ partials in order of arrival. The
    kernel-level tests check the embedding backward itself on fixed rows.)"""
    s = S.ModelShape(1, 2, 128, 50304, 1024)
    B, T = 20, 1024
    flat = S.random_params(s, seed=81)
    idx, tgt = S.zipf_tokens(B, T, 50257, seed=82)
    m = _model(s, "fp32", B, T)
    m.set_params(flat)
    grads = []
    for _ in range(2):
        m.zero_grad()
        m.accumulate(_dev(idx), _dev(tgt), 1.0)
        grads.append(_split(s, m.get_grads())["wte"])
    assert np.array_equal(grads[0], grads[1])
    m.close()


@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_embedding_gradient_two_sort_tiles_matches_oracle(precision):
    """17 x 1024 rows: one full sort tile of 16384 rows and a ragged one of 1024.
    A vocabulary of 256 Zipf ids makes runs from a few rows up to thousands, so
    runs cross 16-entry windows and the tile boundary. The wte gradient is
    compared row by row with the oracle's (each row against its own largest
    element), so that a dropped or doubled embedding row shows even for a rare
    token: fp32 to 1e-4 of the row, bf16 by the row's cosine."""
    s = S.ModelShape(1, 1, 64, 256, 1024)
    B, T = 17, 1024
    idx, tgt = S.zipf_tokens(B, T, s.vocab_size, seed=82)
    flat = S.random_params(s, seed=81)
    P = O.unflatten(_oshape(s), flat.astype(np.float64))
    Mo, Vo = O.zeros_like(_oshape(s)), O.zeros_like(_oshape(s))
    _, _, G = O.train_step(_oshape(s), P, Mo, Vo, 1, idx, tgt, lr=1e-4)
    m = _model(s, precision, B, T)
    m.set_params(flat)
    m.zero_grad()
    m.accumulate(_dev(idx), _dev(tgt), 1.0)
    g, r = _split(s, m.get_grads())["wte"].astype(np.float64), G["wte"]
    counts = np.bincount(idx.ravel(), minlength=s.vocab_size)
    assert counts.min() >= 1 and counts.max() > 16384 // 16
    for v in range(s.vocab_size):
        if precision == "fp32":
            assert np.max(np.abs(g[v] - r[v])) <= 1e-4 * np.max(np.abs(r[v])), (v, counts[v])
        else:
            assert _cos(g[v], r[v]) >= 0.99, (v, counts[v], _cos(g[v], r[v]))
    m.close()


def test_step_graph_replay_matches_eager(monkeypatch):
    """Steps 3+ with one (B, T) replay a captured CUDA graph; a shape change drops
    it. A graph model and an eager model (graphs off) take the same ten steps,
    shape changes included; before each step the graph model is given the eager
    model's parameters and optimiser state, so each step starts from one state.
    Per step: loss 1e-6 and gradient norm 1e-5 relative, gradients 1e-5 of their
    max (not bitwise: the split-K weight-gradient GEMMs add their K partials
    with fp32 atomics, so a gradient's last bits depend on arrival order), and
    the same launch count."""
    s = TINY
    flat = S.random_params(s, seed=31)
    shapes = [(4, 64), (4, 64), (4, 64), (4, 64), (3, 17), (3, 17), (3, 17), (4, 64), (4, 64), (4, 64)]
    monkeypatch.setenv("GPT2_B200_NO_GRAPH", "0")
    mg = _model(s, "bf16", 4, 64)
    monkeypatch.setenv("GPT2_B200_NO_GRAPH", "1")
    me = _model(s, "bf16", 4, 64)
    me.set_params(flat)
    for i, (B, T) in enumerate(shapes):
        mg.set_params(me.get_params())
        m1, v1, t1 = me.get_opt_state()
        mg.set_opt_state(m1, v1, t1)
        idx, tgt = S.uniform_tokens(B, T, s.vocab_size, seed=500 + i)
        lg, ng = mg.step(_dev(idx), _dev(tgt), 3e-4)
        le, ne = me.step(_dev(idx), _dev(tgt), 3e-4)
        assert abs(lg - le) <= 1e-6 * abs(le), (i, lg, le)
        assert abs(ng - ne) <= 1e-5 * abs(ne), (i, ng, ne)
        assert _rel(mg.get_grads(), me.get_grads()) < 1e-5, i
        assert mg.last_launch_count() == me.last_launch_count(), i
    mg.close()
    me.close()


@pytest.mark.parametrize("precision,T", [("fp32", 64), ("fp32", 23), ("bf16", 64), ("bf16", 23)])
def test_forward_last_position_logits(precision, T):
    """gpt2_forward_last: each sequence's last-position logits against the
    oracle's full forward (fp32: 1e-4 of max |logit|; bf16: 2e-2, the bf16
    tolerance), and within 1e-6 of the same row of the GPU's own full-logits
    forward in fp32 mode (the same arithmetic on the same rows)."""
    s = TINY
    B = 3
    idx, _ = S.uniform_tokens(B, T, s.vocab_size, seed=900 + T)
    flat = S.random_params(s, seed=901)
    m = _model(s, precision, 4, 64)
    m.set_params(flat)
    tdt = torch.float32 if precision == "fp32" else torch.bfloat16
    last = torch.empty((B, s.vocab_size), dtype=tdt, device="cuda")
    m.forward_last(_dev(idx), last)
    full = torch.empty((B, T, s.vocab_size), dtype=tdt, device="cuda")
    m.forward(_dev(idx), None, full)
    P = O.unflatten(_oshape(s), flat.astype(np.float64))
    _, ref_logits, _ = O.forward(_oshape(s), P, idx)
    got = last.float().cpu().numpy()
    tol = 1e-4 if precision == "fp32" else 2e-2
    assert _rel(got, ref_logits[:, -1, :]) < tol
    if precision == "fp32":
        assert _rel(got, full[:, -1, :].cpu().numpy()) < 1e-6
    m.close()


# ----------------------------------------------------------------------------
# Layer by layer: every saved activation of a forward against the oracle's
# (the pages' debugging advice: diff each layer's activations).
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("precision", ["fp32", "bf16"])
def test_saved_activations_layer_by_layer(precision):
    """gpt2_debug_activation for every kind and layer against the oracle's forward
    cache (residual states rebuilt from the oracle's cached branch outputs with
    its own linear): fp32 1e-4 of max |value| per tensor, bf16 3e-2 and cosine
    > 0.999."""
    from decoder_only_transformer_sm_b200 import native
    s = TINY
    B, T = 3, 20
    os_ = _oshape(s)
    flat = S.random_params(s, seed=950)
    idx, tgt = S.uniform_tokens(B, T, s.vocab_size, seed=951)
    m = _model(s, precision, 4, 64)
    m.set_params(flat)
    m.forward(_dev(idx), _dev(tgt))
    P = O.unflatten(os_, flat.astype(np.float64))
    _, _, cache = O.forward(os_, P, idx)
    C = s.n_embd

    def flat_heads(z):   # (B, H, T, hd) -> (B, T, C)
        return z.transpose(0, 2, 1, 3).reshape(B, T, C)

    def check(got, ref, what):
        if precision == "fp32":
            assert _rel(got, ref) < 1e-4, what
        else:
            assert _rel(got, ref) < 3e-2, what
            assert _cos(got, ref) > 0.999, what

    x = P["wte"][idx] + P["wpe"][np.arange(T)][None]
    check(m.debug_activation("resid", 0, B, T), x, "resid 0")
    for l in range(s.n_layer):
        c = cache["layers"][l]
        pre = f"h.{l}."
        check(m.debug_activation("ln_1", l, B, T), c["a"], ("ln_1", l))
        qkv = np.concatenate([flat_heads(c["q"]), flat_heads(c["k"]), flat_heads(c["v"])], axis=-1)
        check(m.debug_activation("qkv", l, B, T), qkv, ("qkv", l))
        check(m.debug_activation("attn", l, B, T), c["y"], ("attn", l))
        x = x + O.linear(c["y"], P[pre + "attn.c_proj.weight"], P[pre + "attn.c_proj.bias"])
        check(m.debug_activation("resid", 2 * l + 1, B, T), x, ("resid", 2 * l + 1))
        check(m.debug_activation("ln_2", l, B, T), c["m"], ("ln_2", l))
        check(m.debug_activation("gelu", l, B, T), c["g"], ("gelu", l))
        x = x + O.linear(c["g"], P[pre + "mlp.c_proj.weight"], P[pre + "mlp.c_proj.bias"])
        check(m.debug_activation("resid", 2 * l + 2, B, T), x, ("resid", 2 * l + 2))
    check(m.debug_activation("ln_f", 0, B, T), cache["f"], "ln_f")
    for kind, index in [("ln_1", s.n_layer), ("resid", 2 * s.n_layer + 1), ("ln_f", 1), ("qkv", -1)]:
        with pytest.raises(native.Gpt2Error, match="INVALID_ARG"):
            m.debug_activation(kind, index, B, T)
    m.close()
