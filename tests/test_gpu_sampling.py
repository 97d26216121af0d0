"""Parity of the generation path (key/value-cache decode and sampling) with the
float64 oracle ("GPT-2 from Scratch", "A generation loop").

The oracle recomputes the whole (cropped) sequence for every draw; the CUDA path
fills a key/value cache with a prefill and then runs one position per draw.
  * Decode logits, teacher-forced with seeded tokens, against the oracle's full
    forward at the same positions: fp32 1e-4 of max |logit|, bf16 2e-2 (at 124M:
    3e-2 and cosine > 0.999, the tolerances of the full-size forward check).
  * The newest position's attention against a cache, through the kernel-level
    call, against the oracle's causal attention: fp32 1e-5, bf16 1e-2 of max |out|.
  * Draws: an index decided by floating point on both sides. Where u lies more
    than BAND (1e-4 of the total probability) from both ends of the oracle's
    interval for it, the index must equal the oracle's; inside that band it must
    be an index whose interval reaches within BAND of u and that top-k keeps.
  * Whole generation in fp32 against the oracle's loop: tokens equal up to the
    first draw that falls inside the band (the oracle reports each draw's
    margin; the seeds give 64 of 64 and 9 of 64 clear draws). The first case runs
    all three branches of the loop: the first prefill, decode steps, and the
    re-prefill of the cropped window once the sequence outgrows block_size.
  * bf16 generation, whose draws the bf16 logit error can flip, against the same
    loop composed of the single calls (prefill, decode, sample): equal tokens,
    also across calls that replay the graphed decode step; and
    for the pages' call at 124M, the logits of every one of its 40 draws,
    teacher-forced with the generated tokens, against the oracle's forward.
"""
import numpy as np
import pytest

from oracle import gpt2_oracle as O
from decoder_only_transformer_sm_b200 import synthetic as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TINY = S.TINY                                  # head width 32
TINY64 = S.ModelShape(2, 2, 128, 1024, 64)     # head width 64: tcgen05 attention in bf16
W = S.GPT2_124M
BAND = 1e-4


def _oshape(s):
    return O.Shape(s.n_layer, s.n_head, s.n_embd, s.vocab_size, s.block_size)


def _model(s, precision, B, T, seed=0):
    from decoder_only_transformer_sm_b200 import native
    return native.GPT2(s.n_layer, s.n_head, s.n_embd, s.vocab_size, s.block_size, B, T,
                       precision=precision, seed=seed)


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(float(np.max(np.abs(b))), 1e-30))


def _cos(a, b):
    a = a.astype(np.float64).ravel()
    b = b.astype(np.float64).ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


def _check_draw(j, row64, temperature, top_k, u, band=BAND):
    jo, probs, margin = O.sample_next(row64, temperature, top_k, u)
    if margin > band:
        assert j == jo, (j, jo, margin)
    else:
        assert 0 <= j < len(row64) and probs[j] > 0, j
        cdf = np.cumsum(probs)
        lo = cdf[j - 1] if j > 0 else 0.0
        assert lo - band <= u <= cdf[j] + band, (j, jo, u, lo, cdf[j])


# ----------------------------------------------------------------------------
# The draw (kernel-level call).
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("V", [1000, 50304])
@pytest.mark.parametrize("temperature,top_k", [(1.0, 0), (0.8, 40), (1.3, 1), (0.7, 50), (1.0, 100000)])
def test_sample_kernel_matches_oracle(dtype, V, temperature, top_k):
    from decoder_only_transformer_sm_b200 import native
    rows = 16
    rng = np.random.default_rng(700 + V + top_k)
    x = rng.normal(0.0, 2.0, (rows, V)).astype(np.float32)
    tdt = torch.float32 if dtype == "fp32" else torch.bfloat16
    xd = torch.from_numpy(x).to(tdt).cuda()
    x64 = xd.float().cpu().numpy().astype(np.float64)    # the values both sides see
    u = S.uniforms(1, rows, seed=701 + V)[0]
    nxt = torch.full((rows,), -1, dtype=torch.int32, device="cuda")
    st = native.sample(xd, V, temperature, top_k, torch.from_numpy(u).cuda(), nxt)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got = nxt.cpu().numpy()
    for r in range(rows):
        _check_draw(int(got[r]), x64[r], temperature, top_k, float(u[r]))


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("temperature,top_k", [(1.0, 0), (0.8, 40)])
def test_sample_kernel_long_rows_single_block(dtype, temperature, top_k):
    """Rows of 500,000 values: the slices of an 8-CTA cluster no longer fit its
    shared memory, so the draw runs on one block per row reading the row from
    memory at every pass. Same oracle check as above."""
    from decoder_only_transformer_sm_b200 import native
    rows, V = 3, 500_000
    rng = np.random.default_rng(720 + top_k)
    x = rng.normal(0.0, 2.0, (rows, V)).astype(np.float32)
    tdt = torch.float32 if dtype == "fp32" else torch.bfloat16
    xd = torch.from_numpy(x).to(tdt).cuda()
    x64 = xd.float().cpu().numpy().astype(np.float64)
    u = S.uniforms(1, rows, seed=721)[0]
    nxt = torch.full((rows,), -1, dtype=torch.int32, device="cuda")
    st = native.sample(xd, V, temperature, top_k, torch.from_numpy(u).cuda(), nxt)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got = nxt.cpu().numpy()
    for r in range(rows):
        _check_draw(int(got[r]), x64[r], temperature, top_k, float(u[r]))


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_sample_kernel_ties_row_stride_and_edges(dtype):
    """Integer-valued logits (many ties at the k-th value), a row stride above V,
    an all-equal row, and the u edge cases 0 and just below 1."""
    from decoder_only_transformer_sm_b200 import native
    rows, V, ld = 8, 3000, 3016
    rng = np.random.default_rng(710)
    x = np.round(rng.normal(0.0, 2.0, (rows, ld))).astype(np.float32)
    x[5] = 0.0
    tdt = torch.float32 if dtype == "fp32" else torch.bfloat16
    xd = torch.from_numpy(x).to(tdt).cuda()
    x64 = xd.float().cpu().numpy().astype(np.float64)[:, :V]
    u = S.uniforms(1, rows, seed=711)[0]
    u[0], u[1] = 0.0, np.float32(1.0 - 2.0 ** -24)
    ud = torch.from_numpy(u).cuda()
    for k in (1, 7, 50, V - 1, 0):
        nxt = torch.full((rows,), -1, dtype=torch.int32, device="cuda")
        native.sample(xd, V, 0.9, k, ud, nxt, ld=ld)
        got = nxt.cpu().numpy()
        for r in range(rows):
            j = int(got[r])
            _check_draw(j, x64[r], 0.9, k, float(u[r]))
            if 1 <= k < V:
                kth = np.sort(x64[r])[::-1][k - 1]
                assert x64[r, j] >= kth


def test_sample_argument_errors():
    from decoder_only_transformer_sm_b200 import native
    x = torch.zeros((2, 16), device="cuda")
    u = torch.zeros(2, device="cuda")
    nxt = torch.zeros(2, dtype=torch.int32, device="cuda")
    for temp in (0.0, -1.0, float("inf"), float("nan")):
        with pytest.raises(native.Gpt2Error, match="INVALID_ARG"):
            native.sample(x, 16, temp, 0, u, nxt)
    with pytest.raises(native.Gpt2Error, match="INVALID_ARG"):
        native.sample(x, 16, 1.0, 0, u, nxt, ld=8)


# ----------------------------------------------------------------------------
# Attention of the newest position against the cache (kernel-level call).
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("hd", [64, 32])
@pytest.mark.parametrize("n", [1, 63, 64, 65, 300])
def test_attention_decode_kernel_matches_oracle(dtype, hd, n):
    from decoder_only_transformer_sm_b200 import native
    B, H, Tc = 2, 4, 300
    C = H * hd
    rng = np.random.default_rng(720 + n + hd)
    cache = rng.normal(0.0, 1.0, (B, Tc, 3 * C)).astype(np.float32)
    tdt = torch.float32 if dtype == "fp32" else torch.bfloat16
    cd = torch.from_numpy(cache).to(tdt).cuda()
    c64 = cd.float().cpu().numpy().astype(np.float64)
    out = torch.full((B, C), float("nan"), dtype=tdt, device="cuda")
    ws = torch.zeros(B * H * ((Tc + 63) // 64) * (hd + 2), dtype=torch.float32, device="cuda")
    st = native.attention_decode(cd, out, B, H, hd, Tc, n, ws)
    torch.cuda.synchronize()
    assert int(st.item()) == 0

    def heads(z):
        return z.reshape(B, n, H, hd).transpose(0, 2, 1, 3)

    y, _ = O.causal_attention(heads(c64[:, :n, :C]), heads(c64[:, :n, C:2 * C]), heads(c64[:, :n, 2 * C:]))
    ref = y[:, :, -1, :].reshape(B, C)
    got = out.float().cpu().numpy()
    assert _rel(got, ref) < (1e-5 if dtype == "fp32" else 1e-2)


# ----------------------------------------------------------------------------
# Decode steps against the full forward (teacher forcing with seeded tokens).
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("precision,shape", [("fp32", "tiny"), ("fp32", "tiny64"), ("bf16", "tiny64"),
                                             ("bf16", "tiny")])
def test_decode_logits_match_full_forward(precision, shape):
    s = TINY if shape == "tiny" else TINY64
    B, T0, steps = 3, 10, 20
    flat = S.random_params(s, seed=730)
    seq, _ = S.uniform_tokens(B, T0 + steps, s.vocab_size, seed=731)
    m = _model(s, precision, B, s.block_size)
    m.set_params(flat)
    tdt = torch.float32 if precision == "fp32" else torch.bfloat16
    lg = torch.empty((B, s.vocab_size), dtype=tdt, device="cuda")
    m.prefill(_dev(seq[:, :T0]), lg)
    got = [lg.float().cpu().numpy()]
    for i in range(steps - 1):
        m.decode(_dev(seq[:, T0 + i]), T0 + i, lg)
        got.append(lg.float().cpu().numpy())
    P = O.unflatten(_oshape(s), flat.astype(np.float64))
    _, ref, _ = O.forward(_oshape(s), P, seq[:, :T0 + steps - 1])
    tol = 1e-4 if precision == "fp32" else 2e-2
    for i, g in enumerate(got):
        assert _rel(g, ref[:, T0 - 1 + i, :]) < tol, i
    m.close()


def test_decode_argument_errors():
    from decoder_only_transformer_sm_b200 import native
    s = TINY
    m = _model(s, "fp32", 2, s.block_size)
    lg = torch.empty((2, s.vocab_size), device="cuda")
    tok = _dev(np.zeros(2))
    with pytest.raises(native.Gpt2Error, match="INVALID_ARG"):   # no prefill yet
        m.decode(tok, 1, lg)
    m.prefill(_dev(np.zeros((2, 4))), lg)
    for pos in (0, 5, s.block_size):                            # outside [1, cached length]
        with pytest.raises(native.Gpt2Error, match="INVALID_ARG"):
            m.decode(tok, pos, lg)
    with pytest.raises(native.Gpt2Error, match="INVALID_ARG"):   # more rows than the prefill
        m.decode(_dev(np.zeros(3)), 4, lg)
    m.decode(tok[:1], 4, lg)                                     # one row: row 1 has no entry at 4
    with pytest.raises(native.Gpt2Error, match="INVALID_ARG"):   # so two rows at 5 are refused
        m.decode(tok, 5, lg)
    m.decode(tok[:1], 5, lg)                                     # the next position of row 0 is fine
    m.set_params(m.get_params())                                 # a weight change empties the cache
    with pytest.raises(native.Gpt2Error, match="INVALID_ARG"):
        m.decode(tok[:1], 6, lg)
    out = torch.empty((2, 8), dtype=torch.int32, device="cuda")
    u = torch.zeros((4, 2), device="cuda")
    for temp in (0.0, float("nan")):
        with pytest.raises(native.Gpt2Error, match="INVALID_ARG"):
            m.generate(_dev(np.zeros((2, 4))), 4, temp, 0, u, out)
    m.close()


# ----------------------------------------------------------------------------
# Whole generation.
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("temperature,top_k,clear", [(0.9, 20, 64), (1.0, 0, 9)])
def test_generate_fp32_matches_oracle_loop(temperature, top_k, clear):
    s = TINY
    B, T0, n_new = 2, 5, 64          # 5 + 64 - 1 > block_size: the last draws re-prefill the crop
    flat = S.random_params(s, seed=740, scale=0.2)
    prompt, _ = S.uniform_tokens(B, T0, s.vocab_size, seed=741)
    u = S.uniforms(n_new, B, seed=742)
    m = _model(s, "fp32", B, s.block_size)
    m.set_params(flat)
    out = torch.full((B, T0 + n_new), -1, dtype=torch.int32, device="cuda")
    m.generate(_dev(prompt), n_new, temperature, top_k, torch.from_numpy(u).cuda(), out)
    got = out.cpu().numpy()
    P = O.unflatten(_oshape(s), flat.astype(np.float64))
    ref, margins = O.generate(_oshape(s), P, prompt, n_new, temperature, top_k, u.astype(np.float64))
    close = np.nonzero((margins < BAND).any(axis=1))[0]
    upto = int(close[0]) if close.size else n_new
    assert upto == clear
    assert np.array_equal(got[:, :T0], prompt)
    assert np.array_equal(got[:, :T0 + upto], ref[:, :T0 + upto])
    m.close()


def _composed_loop(m, s, prompt, n_new, temperature, top_k, u_dev, tdt):
    """The generation loop written with the single calls (prefill, decode, sample)."""
    B, T0 = prompt.shape
    seq = np.asarray(prompt, dtype=np.int32).copy()
    lg = torch.empty((B, s.vocab_size), dtype=tdt, device="cuda")
    nxt = torch.empty(B, dtype=torch.int32, device="cuda")
    for step in range(n_new):
        n = T0 + step
        if step == 0 or n > s.block_size:
            w = min(n, s.block_size)
            m.prefill(_dev(seq[:, n - w:n]), lg)
        else:
            m.decode(nxt, n - 1, lg)
        m.sample(lg, temperature, top_k, u_dev[step], nxt)
        seq = np.concatenate([seq, nxt.cpu().numpy()[:, None]], axis=1)
    return seq


def test_generate_bf16_equals_composed_calls():
    s = TINY64
    B, T0, n_new = 3, 7, 62          # crosses block_size = 64
    m = _model(s, "bf16", B, s.block_size, seed=5)
    prompt, _ = S.uniform_tokens(B, T0, s.vocab_size, seed=750)
    u = torch.from_numpy(S.uniforms(n_new, B, seed=751)).cuda()
    out = torch.full((B, T0 + n_new), -1, dtype=torch.int32, device="cuda")
    m.generate(_dev(prompt), n_new, 0.8, 40, u, out)
    ref = _composed_loop(m, s, prompt, n_new, 0.8, 40, u, torch.bfloat16)
    got = out.cpu().numpy()
    assert np.array_equal(got, ref)
    assert got.min() >= 0 and got.max() < s.vocab_size
    m.close()


def test_generate_decode_graph_across_calls():
    """gpt2_generate's decode steps read position, draw index and output slot from
    device arguments and run as one CUDA graph per (B, temperature, top_k): the
    first decode step runs eagerly, the second is captured, later ones replay it,
    and a later call with another (temperature, top_k) starts over. Every call
    must equal the loop of single calls, and a repeated call its first run."""
    s = TINY64
    B, T0, n_new = 2, 3, 20
    m = _model(s, "bf16", B, s.block_size, seed=6)
    prompt, _ = S.uniform_tokens(B, T0, s.vocab_size, seed=752)
    u = torch.from_numpy(S.uniforms(n_new, B, seed=753)).cuda()
    runs = []
    for temperature, top_k in [(0.8, 40), (1.0, 0), (0.8, 40), (0.8, 40)]:
        out = torch.full((B, T0 + n_new), -1, dtype=torch.int32, device="cuda")
        m.generate(_dev(prompt), n_new, temperature, top_k, u, out)
        runs.append(out.cpu().numpy())
    assert np.array_equal(runs[0], _composed_loop(m, s, prompt, n_new, 0.8, 40, u, torch.bfloat16))
    assert np.array_equal(runs[1], _composed_loop(m, s, prompt, n_new, 1.0, 0, u, torch.bfloat16))
    assert np.array_equal(runs[2], runs[0]) and np.array_equal(runs[3], runs[0])
    # a shorter call after a longer one: the draws stop at its own length
    out = torch.full((B, T0 + 5), -1, dtype=torch.int32, device="cuda")
    m.generate(_dev(prompt), 5, 0.8, 40, u, out)
    assert np.array_equal(out.cpu().numpy(), runs[0][:, :T0 + 5])
    m.close()


def _profile_sites(m, fn):
    m.profile(True)
    fn()
    sites = {st["name"] for st in m.profile_read()}
    m.profile(False)
    return sites


@pytest.mark.parametrize("B", [1, 3])
def test_decode_persistent_kernel_matches_kernel_chain(B, monkeypatch):
    """A bf16 decode step of at most four rows runs as one persistent kernel (grid
    barriers between the phases of a layer, weights streamed into shared memory);
    GPT2_B200_NO_MEGA=1 at creation keeps the chain of separate kernels. Same
    weights and cache contents: the logits of five teacher-forced decode steps
    agree to bf16 rounding (1e-2 of max |logit|, cosine > 0.9999), and the profile
    names the kernel that ran."""
    s = TINY64
    seq, _ = S.uniform_tokens(B, 12, s.vocab_size, seed=770 + B)
    out = {}
    for mode in ("mega", "chain"):
        if mode == "chain":
            monkeypatch.setenv("GPT2_B200_NO_MEGA", "1")
        m = _model(s, "bf16", B, s.block_size, seed=7)
        lg = torch.empty((B, s.vocab_size), dtype=torch.bfloat16, device="cuda")
        m.prefill(_dev(seq[:, :6]), lg)
        got = []
        for i in range(5):
            m.decode(_dev(seq[:, 6 + i]), 6 + i, lg)
            got.append(lg.float().cpu().numpy())
        sites = _profile_sites(m, lambda: m.decode(_dev(seq[:, 11]), 11, lg))
        out[mode] = (np.stack(got), sites)
        m.close()
        monkeypatch.delenv("GPT2_B200_NO_MEGA", raising=False)
    assert any("persistent" in x for x in out["mega"][1]), out["mega"][1]
    assert not any("persistent" in x for x in out["chain"][1]), out["chain"][1]
    a, b = out["mega"][0], out["chain"][0]
    assert _rel(a, b) < 1e-2 and _cos(a, b) > 0.9999


# ----------------------------------------------------------------------------
# GPT-2 124M, bf16: the generation workload of the benchmark (B = 1, a short
# prompt, 40 new tokens, temperature 0.8, top-k 40).
# ----------------------------------------------------------------------------
def test_124m_decode_logits_and_generation_loop():
    OS = _oshape(W)
    m = _model(W, "bf16", 2, W.block_size, seed=3)
    flat = S.init_params(W, seed=0)
    m.set_params(flat)
    seq, _ = S.zipf_tokens(2, 12, W.real_vocab, seed=760)
    lg = torch.empty((2, W.vocab_size), dtype=torch.bfloat16, device="cuda")
    m.prefill(_dev(seq[:, :8]), lg)
    got = [lg.float().cpu().numpy()]
    for i in range(3):
        m.decode(_dev(seq[:, 8 + i]), 8 + i, lg)
        got.append(lg.float().cpu().numpy())
    P = O.unflatten(OS, flat)
    _, ref, _ = O.forward(OS, P, seq[:, :11])
    for i, g in enumerate(got):
        for b in range(2):
            r = ref[b, 7 + i]
            assert np.max(np.abs(g[b] - r)) / np.max(np.abs(r)) < 3e-2, (i, b)
            assert _cos(g[b], r) > 0.999, (i, b)
    del P
    prompt = seq[:1, :4]
    u = torch.from_numpy(S.uniforms(40, 1, seed=761)).cuda()
    out = torch.full((1, 44), -1, dtype=torch.int32, device="cuda")
    m.generate(_dev(prompt), 40, 0.8, 40, u, out)
    assert np.array_equal(out.cpu().numpy(), _composed_loop(m, W, prompt, 40, 0.8, 40, u, torch.bfloat16))
    m.close()


def test_124m_pages_call_decode_logits_match_oracle_at_every_step():
    """The pages' sampling call on GPT-2 124M in bf16 (one prompt of 4 tokens, 40
    new tokens, temperature 0.8, top-k 40) through gpt2_generate; then its tokens,
    teacher-forced through prefill + decode, give the logits of all 40 draws, each
    compared with the oracle's forward over the generated sequence at the same
    position (one causal forward gives every prefix's last position): 3e-2 of max
    |logit| and cosine > 0.999, the tolerances of the full-size forward check."""
    OS = _oshape(W)
    m = _model(W, "bf16", 1, W.block_size, seed=3)
    flat = S.init_params(W, seed=0)
    m.set_params(flat)
    prompt = S.zipf_tokens(1, 4, W.real_vocab, seed=1001)[0]
    u = torch.from_numpy(S.uniforms(40, 1, seed=1002)).cuda()
    out = torch.full((1, 44), -1, dtype=torch.int32, device="cuda")
    m.generate(_dev(prompt), 40, 0.8, 40, u, out)
    seq = out.cpu().numpy()
    assert np.array_equal(seq[:, :4], prompt) and seq.min() >= 0 and seq.max() < W.vocab_size
    lg = torch.empty((1, W.vocab_size), dtype=torch.bfloat16, device="cuda")
    m.prefill(_dev(seq[:, :4]), lg)
    got = [lg.float().cpu().numpy()[0]]
    for i in range(39):
        m.decode(_dev(seq[:, 4 + i]), 4 + i, lg)
        got.append(lg.float().cpu().numpy()[0])
    m.close()
    _, ref, _ = O.forward(OS, O.unflatten(OS, flat), seq[:, :43])
    for i, g in enumerate(got):
        r = ref[0, 3 + i]
        assert np.max(np.abs(g - r)) / np.max(np.abs(r)) < 3e-2, i
        assert _cos(g, r) > 0.999, i
