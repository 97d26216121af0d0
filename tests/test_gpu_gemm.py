"""Tensor-core (tcgen05) and SIMT GEMMs through gpt2k_matmul_bf16, against the
oracle's nn.Linear arithmetic (float64) on the same bf16-rounded operands.

Tolerances: fp32 outputs 1e-5 of max|ref| (fp32 accumulation of exact bf16
products over K <= 3072); bf16 outputs 8e-3 of max|ref| (one bf16 rounding,
2^-8 relative, of the stored value)."""
import numpy as np
import pytest

from oracle import gpt2_oracle as O

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

SHAPES = [(256, 256, 128), (296, 200, 72), (1024, 768, 768), (136, 1032, 1000), (8, 8, 8)]


def _bf(shape, g, scale=1.0):
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16).cuda()


def _np(t):
    return t.float().cpu().numpy().astype(np.float64)


def _ref(layout, A, B):
    a, b = _np(A), _np(B)
    if layout == "NT":
        return O.linear(a, b)
    if layout == "NN":
        return O.linear(a, b.T)
    return O.linear(a.T, b.T)


def _operands(layout, M, N, K, g):
    if layout == "NT":
        return _bf((M, K), g), _bf((N, K), g)
    if layout == "NN":
        return _bf((M, K), g), _bf((K, N), g)
    return _bf((K, M), g), _bf((K, N), g)


def _relerr(got, ref):
    return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))


@pytest.mark.parametrize("engine", ["tc", "simt"])
@pytest.mark.parametrize("layout", ["NT", "NN", "TN"])
@pytest.mark.parametrize("shape", SHAPES)
def test_gemm_store_and_accum(engine, layout, shape):
    from decoder_only_transformer_sm_b200 import native
    M, N, K = shape
    g = torch.Generator().manual_seed(M * 7 + N * 3 + K)
    A, B = _operands(layout, M, N, K, g)
    ref = _ref(layout, A, B)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    st = native.matmul_bf16(layout, A, B, M, N, K, "store", out, engine=engine)
    acc0 = torch.randn((M, N), generator=g).cuda()
    acc = acc0.clone()
    native.matmul_bf16(layout, A, B, M, N, K, "accum_f32", acc, beta=1.0, engine=engine, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert _relerr(_np(out), ref) < 8e-3
    assert _relerr(acc.cpu().numpy() - acc0.cpu().numpy(), ref) < 1e-5


@pytest.mark.parametrize("shape", [(296, 200, 72), (1024, 3072, 768)])
def test_gemm_fused_epilogues(shape):
    from decoder_only_transformer_sm_b200 import native
    M, N, K = shape
    g = torch.Generator().manual_seed(11)
    A, B = _operands("NT", M, N, K, g)
    bias = torch.randn(N, generator=g).cuda()
    ref = _ref("NT", A, B) + bias.cpu().numpy()
    # bias
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    native.matmul_bf16("NT", A, B, M, N, K, "bias", out, bias=bias)
    # bias + gelu: out = gelu(u), out2 = gelu'(u), u = bias + acc rounded to bf16
    g_out = torch.empty_like(out)
    d_out2 = torch.empty_like(out)
    native.matmul_bf16("NT", A, B, M, N, K, "bias_gelu", g_out, out2=d_out2, bias=bias)
    # bias + residual (fp32)
    resid = torch.randn((M, N), generator=g).cuda()
    r_out = torch.empty((M, N), dtype=torch.float32, device="cuda")
    native.matmul_bf16("NT", A, B, M, N, K, "bias_resid", r_out, bias=bias, resid=resid)
    # multiply by a stored factor (the GELU backward)
    aux = torch.randn((M, N), generator=g).to(torch.bfloat16).cuda()
    m_out = torch.empty_like(out)
    native.matmul_bf16("NT", A, B, M, N, K, "mul", m_out, aux=aux)
    torch.cuda.synchronize()
    assert _relerr(_np(out), ref) < 8e-3
    u = _np(out)                       # bf16-rounded pre-activation
    assert _relerr(_np(g_out), O.gelu_tanh(u)) < 8e-3
    assert _relerr(_np(d_out2), O.gelu_tanh_grad(u)) < 8e-3
    assert _relerr(r_out.cpu().numpy(), resid.cpu().numpy() + ref) < 1e-5
    assert _relerr(_np(m_out), _ref("NT", A, B) * _np(aux)) < 8e-3


@pytest.mark.parametrize("shape", [(296, 200, 72), (1000, 3072, 768), (16384, 3072, 768)])
def test_gemm_mul_column_sums(shape):
    """GPT2K_EPI_MUL with colsum_part: per 32-row group, the column sums of the
    stored bf16 results (checked against sums of the stored output itself, so
    only summation order separates the two: 1e-5 of the group's absolute sum)."""
    from decoder_only_transformer_sm_b200 import native
    M, N, K = shape
    g = torch.Generator().manual_seed(5)
    A, B = _operands("NN", M, N, K, g)
    aux = torch.randn((M, N), generator=g).to(torch.bfloat16).cuda()
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ng = (M + 31) // 32
    part = torch.full((ng, N), float("nan"), device="cuda")
    st = native.matmul_bf16("NN", A, B, M, N, K, "mul", out, aux=aux, colsum_part=part)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    o = _np(out)
    pad = np.zeros((ng * 32, N))
    pad[:M] = o
    ref = pad.reshape(ng, 32, N).sum(axis=1)
    scale = np.abs(pad).reshape(ng, 32, N).sum(axis=1) + 1e-30
    got = part.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(got - ref) / scale) < 1e-5
    assert _relerr(o, _ref("NN", A, B) * _np(aux)) < 8e-3


def test_colsum_needs_tc_mul():
    from decoder_only_transformer_sm_b200 import native
    A = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    part = torch.zeros((2, 64), device="cuda")
    with pytest.raises(native.Gpt2Error):
        native.matmul_bf16("NT", A, A, 64, 64, 64, "store", out, colsum_part=part)
    with pytest.raises(native.Gpt2Error):
        native.matmul_bf16("NT", A, A, 64, 64, 64, "mul", out, aux=A, colsum_part=part, engine="simt")


def test_tc_rejects_unaligned_shapes():
    from decoder_only_transformer_sm_b200 import native
    A = torch.zeros((16, 12), dtype=torch.bfloat16, device="cuda")
    B = torch.zeros((16, 12), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((16, 16), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(native.Gpt2Error):
        native.matmul_bf16("NT", A, B, 16, 16, 12, "store", out, engine="tc")
