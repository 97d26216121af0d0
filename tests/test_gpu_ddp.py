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
