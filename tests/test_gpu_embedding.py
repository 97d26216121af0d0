"""Embedding backward through gpt2k_embedding_bwd against the oracle's
embedding_backward (the transposed selection of "Embeddings: tokens and
positions", "GPT-2 from Scratch").

Exact cases: the rows of dx (and the starting gradients) are small integers
times 2^-10, so every partial sum of at most 2^17 such rows is an fp32 number
and the result is exact in any summation order: the GPU result must equal the
oracle's bit for bit, on the ordered path and on the atomic one. A dropped,
doubled or misplaced row changes some element. Float cases (normal rows): the
ordered path gives bit-identical results on repeated calls, and each token's
row is within 1e-5 of that row's largest element of the oracle's."""
import numpy as np
import pytest

from oracle import gpt2_oracle as O
from decoder_only_transformer_sm_b200 import synthetic as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _ids(kind, B, T, V, seed):
    if kind == "zipf":
        return S.zipf_tokens(B, T, V, seed=seed)[0]
    rng = np.random.default_rng(seed)
    if kind == "one":                       # a single run through every window and chunk
        return np.full((B, T), V // 2, dtype=np.int32)
    if kind == "distinct":                  # no repeats at all
        return rng.permutation(V)[:B * T].reshape(B, T).astype(np.int32)
    return rng.integers(0, V, size=(B, T)).astype(np.int32)


def _run(idx, dx, dwte0, dwpe0, workspace):
    from decoder_only_transformer_sm_b200 import native
    B, T = idx.shape
    C = dx.shape[-1]
    d_idx = torch.from_numpy(np.ascontiguousarray(idx, dtype=np.int32)).cuda()
    d_dx = torch.from_numpy(np.ascontiguousarray(dx.reshape(B * T, C), dtype=np.float32)).cuda()
    d_wte = torch.from_numpy(dwte0.astype(np.float32)).cuda()
    d_wpe = torch.from_numpy(dwpe0.astype(np.float32)).cuda()
    ws = None
    if workspace:
        ws = torch.empty(native.embedding_bwd_workspace(B, T, C), dtype=torch.float32, device="cuda")
    status = native.embedding_bwd(d_idx, d_dx, d_wte, d_wpe, B, T, workspace=ws)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return d_wte.cpu().numpy(), d_wpe.cpu().numpy()


def _exact_inputs(idx, V, C, seed):
    rng = np.random.default_rng(seed)
    B, T = idx.shape
    dx = rng.integers(-8, 9, size=(B, T, C)).astype(np.float64) * 2.0 ** -10
    dwte0 = rng.integers(-8, 9, size=(V, C)).astype(np.float64) * 2.0 ** -10
    dwpe0 = rng.integers(-8, 9, size=(T, C)).astype(np.float64) * 2.0 ** -10
    return dx, dwte0, dwpe0


# (B, T, C, V, ids): the 124M width and vocabulary over two sort tiles (the second
# ragged); one full tile; a one-row second tile; the widths of medium, large (C =
# 1280: 10 lane groups) and XL (1600: a partial lane group); the widest ordered
# width (2048) and one past it (atomic); a vocabulary past 65536 ids (atomic);
# a width that is not a multiple of 128; one row; one id everywhere; no repeats.
EXACT = [
    (17, 1024, 768, 50304, "zipf"),
    (16, 1024, 768, 50304, "zipf"),
    (1, 16385, 64, 1000, "zipf"),
    (4, 1024, 1024, 50304, "zipf"),
    (3, 700, 1280, 4096, "uniform"),
    (2, 1024, 1600, 50304, "zipf"),
    (2, 512, 2048, 8192, "zipf"),
    (2, 512, 2052, 8192, "zipf"),
    (4, 1024, 256, 70000, "zipf"),
    (3, 333, 100, 500, "uniform"),
    (1, 1, 768, 50304, "uniform"),
    (9, 2000, 64, 50304, "one"),
    (4, 1000, 128, 50304, "distinct"),
]


@pytest.mark.parametrize("workspace", [True, False])
@pytest.mark.parametrize("case", EXACT, ids=lambda c: "x".join(map(str, c)))
def test_embedding_bwd_exact(case, workspace):
    B, T, C, V, kind = case
    idx = _ids(kind, B, T, V, seed=90 + B + T)
    dx, dwte0, dwpe0 = _exact_inputs(idx, V, C, seed=91 + C)
    rw, rp = O.embedding_backward(idx, dx, V, T)
    g_wte, g_wpe = _run(idx, dx, dwte0, dwpe0, workspace)
    assert np.array_equal(g_wte, (dwte0 + rw).astype(np.float32))
    assert np.array_equal(g_wpe, (dwpe0 + rp).astype(np.float32))


@pytest.mark.parametrize("case", [(17, 1024, 768, 50304), (2, 1024, 1600, 50304), (6, 1024, 2048, 30000)])
def test_embedding_bwd_ordered_is_deterministic_and_close(case):
    B, T, C, V = case
    idx = _ids("zipf", B, T, V, seed=92)
    rng = np.random.default_rng(93)
    dx = rng.normal(size=(B, T, C))
    z_wte, z_wpe = np.zeros((V, C)), np.zeros((T, C))
    a = _run(idx, dx, z_wte, z_wpe, True)
    b = _run(idx, dx, z_wte, z_wpe, True)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    rw, rp = O.embedding_backward(idx, dx.astype(np.float32).astype(np.float64), V, T)
    used = np.unique(idx)
    err = np.max(np.abs(a[0][used] - rw[used]), axis=1)
    scale = np.max(np.abs(rw[used]), axis=1)
    assert np.all(err <= 1e-5 * scale), float(np.max(err / scale))
    assert not a[0][np.setdiff1d(np.arange(V), used)].any()
    assert np.max(np.abs(a[1] - rp)) <= 1e-5 * np.max(np.abs(rp))

