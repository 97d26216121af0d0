"""Data parallelism (decoder_only_transformer_sm_b200.ddp) as two gloo ranks on
CPU, with an oracle-backed stand-in for the library's model (the same five
calls). After broadcast_params and two DataParallel steps, each rank on its own
two micro-batches, both ranks must hold identical parameters, equal (float64
rounding apart) to one process accumulating all four micro-batches with
loss scale 1/4 and updating ("How to scale up"; "Scaling to 8 GPUs with
DistributedDataParallel": the averaged gradient equals the gradient of the
combined batch). Rendezvous on 127.0.0.1."""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import gpt2_oracle as O
from decoder_only_transformer_sm_b200 import synthetic as S

MICRO = O.Shape(n_layer=2, n_head=2, n_embd=16, vocab_size=64, block_size=8)
LR = 6e-4


class OracleModel:
    """The model interface DataParallel drives, computed by the float64 oracle."""

    def __init__(self, s, flat):
        self.s = s
        self.P = O.unflatten(s, flat)
        self.M, self.V = O.zeros_like(s), O.zeros_like(s)
        self.t = 0
        self.g = torch.zeros(len(flat), dtype=torch.float64)
        self.loss = 0.0

    def zero_grad(self):
        self.g.zero_()
        self.loss = 0.0

    def accumulate(self, idx, targets, loss_scale):
        loss, _, cache = O.forward(self.s, self.P, idx, targets)
        G = O.backward(self.s, self.P, cache, loss_scale=loss_scale)
        self.g += torch.from_numpy(O.flatten(self.s, G))
        self.loss += loss_scale * loss

    def grads_view(self):
        return self.g

    def grad_buckets(self):
        """The flat layout's ranges in the order a backward finishes them: ln_f,
        the blocks from the last to the first, then wte and wpe."""
        offs, o = {}, 0
        for name, shp in O.layout(self.s):
            offs[name] = o
            o += int(np.prod(shp))
        L = self.s.n_layer
        start = [offs[f"h.{l}.ln_1.weight"] for l in range(L)] + [offs["ln_f.weight"]]
        out = [(offs["ln_f.weight"], o - offs["ln_f.weight"])]
        out += [(start[l], start[l + 1] - start[l]) for l in range(L - 1, -1, -1)]
        out.append((0, start[0]))
        return out

    def update(self, lr):
        G = O.unflatten(self.s, self.g.numpy())
        self.t += 1
        norm = O.adamw_update(self.s, self.P, G, self.M, self.V, self.t, lr)
        return self.loss, norm

    def get_params(self):
        return O.flatten(self.s, self.P)

    def set_params(self, flat):
        self.P = O.unflatten(self.s, np.asarray(flat, dtype=np.float64))


def _syn(s):
    return S.ModelShape(s.n_layer, s.n_head, s.n_embd, s.vocab_size, s.block_size)


def _batches(rank):
    out = []
    for k in range(2):
        idx, tgt = S.uniform_tokens(2, 8, MICRO.vocab_size, seed=900 + 10 * rank + k)
        if k == 1:
            tgt[0, :3] = -1     # masked targets change the per-micro-batch mean
        out.append((idx, tgt))
    return out


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir, bucketed):
    import torch.distributed as dist
    from decoder_only_transformer_sm_b200.ddp import DataParallel
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank 1 starts from other weights: broadcast_params must replace them
        flat = S.random_params(_syn(MICRO), seed=77 + rank).astype(np.float64)
        dp = DataParallel(OracleModel(MICRO, flat), bucketed=bucketed)
        assert (dp.buckets is not None) == bucketed
        dp.broadcast_params()
        res = [dp.step(_batches(rank), LR) for _ in range(2)]
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), params=dp.model.get_params(),
                 losses=[r[0] for r in res], norms=[r[1] for r in res])
    finally:
        dist.destroy_process_group()


def test_oracle_model_buckets_partition_the_gradient():
    m = OracleModel(MICRO, S.random_params(_syn(MICRO), seed=1).astype(np.float64))
    b = m.grad_buckets()
    assert len(b) == MICRO.n_layer + 2
    assert sum(c for _, c in b) == len(m.g)
    ends = sorted(b)
    assert all(ends[i][0] + ends[i][1] == ends[i + 1][0] for i in range(len(ends) - 1))
    assert b[-1][0] == 0 and b[0][0] + b[0][1] == len(m.g)      # wte/wpe last, ln_f first


@pytest.mark.parametrize("bucketed", [True, False])
def test_two_ranks_equal_one_process_over_the_combined_batches(tmp_path, bucketed):
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path), bucketed), nprocs=world,
                       start_method="spawn")
    r = [np.load(tmp_path / f"r{k}.npz") for k in range(world)]
    assert np.array_equal(r[0]["params"], r[1]["params"])          # the replicas stay identical
    assert np.array_equal(r[0]["losses"], r[1]["losses"])
    # one process, all four micro-batches accumulated with scale 1/4
    s = MICRO
    P = O.unflatten(s, S.random_params(_syn(s), seed=77).astype(np.float64))
    M, V = O.zeros_like(s), O.zeros_like(s)
    all_batches = _batches(0) + _batches(1)
    for t in (1, 2):
        loss, G = O.accumulate_grads(s, P, all_batches)
        norm = O.adamw_update(s, P, G, M, V, t, LR)
        assert r[0]["losses"][t - 1] == pytest.approx(loss, rel=1e-12)
        assert r[0]["norms"][t - 1] == pytest.approx(norm, rel=1e-12)
    assert np.max(np.abs(r[0]["params"] - O.flatten(s, P))) < 1e-12


def test_single_process_group_is_a_plain_step(tmp_path):
    """world = 1: no collective; the step equals the oracle's accumulate + update."""
    import torch.distributed as dist
    from decoder_only_transformer_sm_b200.ddp import DataParallel
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        flat = S.random_params(_syn(MICRO), seed=78).astype(np.float64)
        dp = DataParallel(OracleModel(MICRO, flat))
        loss, norm = dp.step(_batches(0), LR)
        P = O.unflatten(MICRO, flat)
        ref_loss, G = O.accumulate_grads(MICRO, P, _batches(0))
        assert loss == pytest.approx(ref_loss, rel=1e-12)
        assert norm == pytest.approx(O.grad_norm(G), rel=1e-12)
        with pytest.raises(ValueError):
            dp.step([], LR)
    finally:
        dist.destroy_process_group()
