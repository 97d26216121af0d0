"""Attention kernels through gpt2k_attention_fwd/bwd against the oracle's
causal_attention / causal_attention_backward (float64, materialised T x T).

Tolerances (max|gpu - ref| / max|ref| per tensor): fp32 1e-4; bf16 operands
2e-2 (outputs and gradients are stored in bf16, 2^-8 relative)."""
import numpy as np
import pytest

from oracle import gpt2_oracle as O

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

# the last two have more 128-query work items (B*H*ceil(T/128) = 256, 576) than
# a B200 has SMs, so the persistent kernels walk several items per CTA
CASES = [(2, 64, 4, 32), (3, 37, 2, 64), (1, 1, 3, 64), (2, 200, 12, 64), (1, 1024, 2, 64),
         (2, 1000, 16, 64), (3, 300, 64, 64)]


def _heads(x, B, T, H, hd):
    return x.reshape(B, T, H, hd).transpose(0, 2, 1, 3)


def _merge(x, B, T, H, hd):
    return x.transpose(0, 2, 1, 3).reshape(B, T, H * hd)


def _rel(a, b):
    # floor 1e-3 (inputs are O(1)): at T = 1 the exact dQ is identically zero
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-3))


@pytest.mark.parametrize("dtype,engine", [("fp32", 0), ("bf16", 0), ("bf16", 1), ("bf16", 2)])
@pytest.mark.parametrize("case", CASES + [(2, 300, 3, 64), (1, 129, 1, 64)])
def test_attention_fwd_bwd_vs_oracle(dtype, engine, case):
    from decoder_only_transformer_sm_b200 import native
    B, T, H, hd = case
    if engine == 2 and hd != 64:
        pytest.skip("the tcgen05 engine is for head width 64")
    C = H * hd
    tdt = torch.float32 if dtype == "fp32" else torch.bfloat16
    g = torch.Generator().manual_seed(B * 1000 + T * 10 + H)
    qkv = torch.randn((B, T, 3 * C), generator=g).to(tdt).cuda()
    dout = torch.randn((B, T, C), generator=g).to(tdt).cuda()
    out = torch.empty((B, T, C), dtype=tdt, device="cuda")
    lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    dqkv = torch.empty_like(qkv)
    ws = torch.empty((native.attention_bwd_workspace(B, T, H, hd, engine),), dtype=torch.float32, device="cuda")
    st = native.attention_fwd(qkv, out, lse, B, T, H, hd, engine=engine)
    native.attention_bwd(qkv, out, dout, lse, dqkv, B, T, H, hd, ws, engine=engine, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    x = qkv.float().cpu().numpy().astype(np.float64)
    q, k, v = (_heads(x[..., i * C:(i + 1) * C], B, T, H, hd) for i in range(3))
    y, p = O.causal_attention(q, k, v)
    tol = 1e-4 if dtype == "fp32" else 2e-2
    assert _rel(out.float().cpu().numpy(), _merge(y, B, T, H, hd)) < tol
    ref_lse = np.log(np.sum(np.exp((q @ k.transpose(0, 1, 3, 2)) / np.sqrt(hd)
                                   + np.triu(np.full((T, T), -np.inf), 1)), axis=-1))
    assert np.max(np.abs(lse.cpu().numpy() - ref_lse)) < (1e-4 if dtype == "fp32" else 2e-2)
    # backward against the oracle, fed the kernel's own (rounded) output gradient
    do = _heads(dout.float().cpu().numpy().astype(np.float64), B, T, H, hd)
    dq, dk, dv = O.causal_attention_backward(do, q, k, v, p)
    got = dqkv.float().cpu().numpy()
    for i, ref in enumerate((dq, dk, dv)):
        assert _rel(got[..., i * C:(i + 1) * C], _merge(ref, B, T, H, hd)) < tol, i


@pytest.mark.parametrize("case", [(2, 200, 12, 64), (3, 37, 2, 64), (1, 1, 3, 64), (16, 1024, 12, 64)])
def test_tcgen05_backward_column_sums(case):
    """colsum_part of the tcgen05 backward: per sequence and 32-row group, the
    column sums of the stored dqkv rows (compared with sums of the stored dqkv
    itself, so only the summation order separates them: 1e-5 of the group's
    absolute sum); ragged T leaves a short last group."""
    from decoder_only_transformer_sm_b200 import native
    B, T, H, hd = case
    C = H * hd
    g = torch.Generator().manual_seed(7 * T + H)
    qkv = torch.randn((B, T, 3 * C), generator=g).to(torch.bfloat16).cuda()
    dout = torch.randn((B, T, C), generator=g).to(torch.bfloat16).cuda()
    out = torch.empty((B, T, C), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    dqkv = torch.empty_like(qkv)
    ws = torch.empty((native.attention_bwd_workspace(B, T, H, hd, 2),), dtype=torch.float32, device="cuda")
    G = (T + 31) // 32
    part = torch.full((B * G, 3 * C), float("nan"), device="cuda")
    st = native.attention_fwd(qkv, out, lse, B, T, H, hd, engine=2)
    native.attention_bwd(qkv, out, dout, lse, dqkv, B, T, H, hd, ws, engine=2, status=st, colsum_part=part)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    d = dqkv.float().cpu().numpy().astype(np.float64)
    pad = np.zeros((B, G * 32, 3 * C))
    pad[:, :T] = d
    ref = pad.reshape(B * G, 32, 3 * C).sum(axis=1)
    scale = np.abs(pad).reshape(B * G, 32, 3 * C).sum(axis=1) + 1e-30
    got = part.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(got - ref) / scale) < 1e-5


def test_column_sums_need_tcgen05_backward():
    from decoder_only_transformer_sm_b200 import native
    B, T, H, hd = 1, 64, 1, 64
    x = torch.zeros((B, T, 3 * H * hd), dtype=torch.bfloat16, device="cuda")
    o = torch.zeros((B, T, H * hd), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((B, H, T), device="cuda")
    ws = torch.zeros(B * H * T, device="cuda")
    part = torch.zeros((2, 3 * H * hd), device="cuda")
    with pytest.raises(native.Gpt2Error):
        native.attention_bwd(x, o, o, lse, torch.zeros_like(x), B, T, H, hd, ws, engine=1, colsum_part=part)


def test_attention_rejects_bad_head_width():
    from decoder_only_transformer_sm_b200 import native
    x = torch.zeros((1, 4, 3 * 48), device="cuda")
    with pytest.raises(native.Gpt2Error):
        native.attention_fwd(x, torch.zeros((1, 4, 48), device="cuda"), torch.zeros((1, 1, 4), device="cuda"),
                             1, 4, 1, 48)
