"""The data-parallel pieces on one GPU: the gradient buffer view shares the
library's memory, and an NCCL all-reduce over one rank on that view, followed by
the update, equals a plain step. (Two or more GPUs are not available to these
tests; the two-rank arithmetic is tested with gloo on CPU in test_ddp_cpu.py.)"""
import os
import socket

import numpy as np
import pytest

from decoder_only_transformer_sm_b200 import synthetic as S

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

TINY = S.TINY


def _model(precision="fp32", seed=0):
    from decoder_only_transformer_sm_b200 import native
    s = TINY
    return native.GPT2(s.n_layer, s.n_head, s.n_embd, s.vocab_size, s.block_size, 2, 32,
                       precision=precision, seed=seed)


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def test_grads_view_shares_the_gradient_buffer():
    m = _model()
    m.set_params(S.random_params(TINY, seed=60))
    idx, tgt = S.uniform_tokens(2, 32, TINY.vocab_size, seed=61)
    m.zero_grad()
    m.accumulate(_dev(idx), _dev(tgt), 1.0)
    g = m.grads_view()
    torch.cuda.synchronize()
    assert g.dtype == torch.float32 and g.numel() == m.n_params and g.is_cuda
    assert np.array_equal(g.cpu().numpy(), m.get_grads())
    g.mul_(0.5)                               # a write through the view reaches the library
    torch.cuda.synchronize()
    assert np.array_equal(g.cpu().numpy(), m.get_grads())
    m.close()


def test_single_rank_nccl_allreduce_then_update_equals_step():
    import torch.distributed as dist
    from decoder_only_transformer_sm_b200.ddp import DataParallel
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        flat = S.random_params(TINY, seed=62)
        idx, tgt = S.uniform_tokens(2, 32, TINY.vocab_size, seed=63)
        a, b = _model(), _model()
        a.set_params(flat)
        b.set_params(flat)
        dp = DataParallel(a)
        dp.broadcast_params()
        a.zero_grad()
        a.accumulate(_dev(idx), _dev(tgt), 1.0)
        before = a.get_grads()
        dist.all_reduce(a.grads_view())       # the collective on the library's buffer (one rank: identity)
        torch.cuda.synchronize()
        assert np.array_equal(a.get_grads(), before)
        loss_a, norm_a = a.update(6e-4)
        loss_b, norm_b = b.step(_dev(idx), _dev(tgt), 6e-4)
        assert loss_a == pytest.approx(loss_b, rel=1e-6)
        assert norm_a == pytest.approx(norm_b, rel=1e-5)
        gb = b.get_grads()
        assert np.max(np.abs(before - gb)) <= 1e-5 * np.max(np.abs(gb))
        # the embedding backward adds with atomics: a gradient within rounding of
        # zero can change sign, and AdamW's first step then moves that element by 2 lr
        d = np.abs(a.get_params() - b.get_params())
        assert d.max() < 2.5 * 6e-4
        assert np.mean(d < 1e-6) > 0.9999
        loss_c, _ = dp.step([(_dev(idx), _dev(tgt))], 6e-4)   # the wrapper's own step
        assert np.isfinite(loss_c)
        a.close()
        b.close()
    finally:
        dist.destroy_process_group()


def test_grad_buckets_follow_the_backward_order():
    """gpt2_grad_buckets: ln_f, blocks n_layer-1 .. 0, then wte and wpe; together
    they cover the flat gradient vector once."""
    from oracle import gpt2_oracle as O
    m = _model()
    b = m.grad_buckets()
    s = TINY
    offs, o = {}, 0
    for name, shp in O.layout(O.Shape(s.n_layer, s.n_head, s.n_embd, s.vocab_size, s.block_size)):
        offs[name] = o
        o += int(np.prod(shp))
    assert o == m.n_params and len(b) == s.n_layer + 2
    assert b[0] == (offs["ln_f.weight"], m.n_params - offs["ln_f.weight"])
    for k, l in enumerate(range(s.n_layer - 1, -1, -1), start=1):
        end = offs[f"h.{l + 1}.ln_1.weight"] if l + 1 < s.n_layer else offs["ln_f.weight"]
        assert b[k] == (offs[f"h.{l}.ln_1.weight"], end - offs[f"h.{l}.ln_1.weight"])
    assert b[-1] == (0, offs["h.0.ln_1.weight"])
    m.close()


def test_bucketed_exchange_on_one_nccl_rank_equals_step():
    """The bucketed exchange on a one-rank NCCL group: the library records one
    event per bucket in the backward, the communication stream waits for each and
    all-reduces that bucket (the identity over one rank), the update waits for
    the communication stream; the result equals a plain step."""
    import torch.distributed as dist
    from decoder_only_transformer_sm_b200.ddp import DataParallel
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        flat = S.random_params(TINY, seed=64)
        idx, tgt = S.uniform_tokens(2, 32, TINY.vocab_size, seed=65)
        a, b = _model("bf16"), _model("bf16")
        a.set_params(flat)
        b.set_params(flat)
        dp = DataParallel(a)
        assert dp.buckets == a.grad_buckets() and dp.comm is not None and len(dp.events) == len(dp.buckets)
        for step in range(2):
            a.zero_grad()
            a.accumulate(_dev(idx), _dev(tgt), 1.0)
            dp._exchange(a.grads_view())
            torch.cuda.current_stream().synchronize()
            assert all(ev.query() for ev in dp.events)
            loss_a, norm_a = a.update(6e-4)
            loss_b, norm_b = b.step(_dev(idx), _dev(tgt), 6e-4)
            assert loss_a == pytest.approx(loss_b, rel=1e-6)
            assert norm_a == pytest.approx(norm_b, rel=1e-5)
        a.set_grad_events(None)
        a.close()
        b.close()
    finally:
        dist.destroy_process_group()
