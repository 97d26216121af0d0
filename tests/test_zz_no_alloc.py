"""The attention backward variant that allocates nothing
(gpt2k_attention_bwd_noalloc), for callers that cannot call cudaMalloc: its
output must match gpt2k_attention_bwd (caller-allocated workspace) within the
attention tests' tolerance, on two calls in a row (the second with another
shape, so it runs on the array the first call left behind).

This file sorts last so that a run stopping at its first failure has already
run every other test."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-4, "bf16": 2e-2}


def _inputs(B, T, H, hd, tdt, seed):
    from decoder_only_transformer_sm_b200 import native
    C = H * hd
    g = torch.Generator().manual_seed(seed)
    qkv = torch.randn((B, T, 3 * C), generator=g).to(tdt).cuda()
    dout = torch.randn((B, T, C), generator=g).to(tdt).cuda()
    out = torch.empty((B, T, C), dtype=tdt, device="cuda")
    lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    native.attention_fwd(qkv, out, lse, B, T, H, hd)
    return qkv, out, dout, lse


def _rel(a, b):
    a = a.float().cpu().numpy()
    b = b.float().cpu().numpy()
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_noalloc_matches_workspace_variant_twice(dtype):
    from decoder_only_transformer_sm_b200 import native
    tdt = torch.float32 if dtype == "fp32" else torch.bfloat16
    for call, (B, T, H, hd) in enumerate([(4, 1024, 12, 64), (3, 37, 4, 32)]):
        qkv, out, dout, lse = _inputs(B, T, H, hd, tdt, seed=100 + call)
        ref = torch.empty_like(qkv)
        ws = torch.empty((B * H * T,), dtype=torch.float32, device="cuda")
        st = native.attention_bwd(qkv, out, dout, lse, ref, B, T, H, hd, ws)
        got = torch.full_like(qkv, float("nan"))
        torch.cuda.synchronize()
        free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
        native.attention_bwd_noalloc(qkv, out, dout, lse, got, B, T, H, hd, status=st)
        torch.cuda.synchronize()
        if call == 1:   # the first call may load the module; the second must allocate nothing
            assert torch.cuda.mem_get_info()[0] == free0
            assert torch.cuda.memory_allocated() == alloc0
        assert int(st.item()) == 0
        assert torch.isfinite(got.float()).all()
        assert _rel(got, ref) <= TOL[dtype], (call, _rel(got, ref))


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from decoder_only_transformer_sm_b200 import native
    B, T, H, hd = 2, 1024, 129, 32          # B*H*T = 264192 > 262144
    x = torch.zeros((1,), dtype=torch.float32, device="cuda")
    with pytest.raises(native.Gpt2Error) as e:
        native.attention_bwd_noalloc(x, x, x, x, x, B, T, H, hd)
    assert e.value.code == -1 and "262144" in str(e.value)
