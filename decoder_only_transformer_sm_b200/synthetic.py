"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module holds only random draws and the parameter naming/shape list; it
contains none of the model's arithmetic (no forward, loss, backward or update).

* Parameter names and shapes follow the module tree of "GPT-2 from Scratch",
  sections "Embeddings: tokens and positions", "CausalSelfAttention",
  "The MLP and GPT-2's GELU", "The Block: pre-LN and residuals" and
  "The full model" (wte, wpe, h.{l}.{ln_1, attn.c_attn, attn.c_proj, ln_2,
  mlp.c_fc, mlp.c_proj}, ln_f; lm_head is wte itself).
* The initial weights are the random draw of "GPT-2 from Scratch",
  "Initialization: 0.02, and the residual scaling": N(0, 0.02) for Linear and
  Embedding weights, N(0, 0.02/sqrt(2*n_layer)) for every ``*.c_proj.weight``,
  zero biases, LayerNorm weight 1 and bias 0.
* Token streams stand in for the pages' corpora (FineWeb-Edu, tiny
  Shakespeare), which are not available: uniform ids for the tiny config and a
  truncated Zipf(1.1) law over the real GPT-2 ids for the large ones, with
  targets the same stream shifted by one ("The data loader with the
  shift-by-one").
"""
from __future__ import annotations

from dataclasses import dataclass
import math

import numpy as np


@dataclass(frozen=True)
class ModelShape:
    n_layer: int
    n_head: int
    n_embd: int
    vocab_size: int      # rows of wte (padded vocabulary)
    block_size: int      # rows of wpe
    vocab_real: int = 0  # ids actually drawn; 0 means vocab_size

    @property
    def real_vocab(self) -> int:
        return self.vocab_real or self.vocab_size


# The workloads of this repository (name -> shape, batch, seed, token law).
TINY = ModelShape(n_layer=2, n_head=4, n_embd=128, vocab_size=1024, block_size=64)
GPT2_124M = ModelShape(12, 12, 768, 50304, 1024, 50257)
GPT2_MEDIUM = ModelShape(24, 16, 1024, 50304, 1024, 50257)
GPT2_XL = ModelShape(48, 25, 1600, 50304, 1024, 50257)


def param_layout(s: ModelShape):
    """Ordered list of (name, shape, is_2d). The tied lm_head is listed once (as wte)."""
    C, V = s.n_embd, s.vocab_size
    out = [("wte", (V, C)), ("wpe", (s.block_size, C))]
    for l in range(s.n_layer):
        p = f"h.{l}."
        out += [
            (p + "ln_1.weight", (C,)), (p + "ln_1.bias", (C,)),
            (p + "attn.c_attn.weight", (3 * C, C)), (p + "attn.c_attn.bias", (3 * C,)),
            (p + "attn.c_proj.weight", (C, C)), (p + "attn.c_proj.bias", (C,)),
            (p + "ln_2.weight", (C,)), (p + "ln_2.bias", (C,)),
            (p + "mlp.c_fc.weight", (4 * C, C)), (p + "mlp.c_fc.bias", (4 * C,)),
            (p + "mlp.c_proj.weight", (C, 4 * C)), (p + "mlp.c_proj.bias", (C,)),
        ]
    out += [("ln_f.weight", (C,)), ("ln_f.bias", (C,))]
    return [(n, shp, len(shp) == 2) for n, shp in out]


def num_params(s: ModelShape) -> int:
    return sum(int(np.prod(shp)) for _, shp, _ in param_layout(s))


def init_params(s: ModelShape, seed: int = 0, dtype=np.float32) -> np.ndarray:
    """Flat parameter vector in ``param_layout`` order, drawn with default_rng(seed)."""
    rng = np.random.default_rng(seed)
    chunks = []
    resid_std = 0.02 / math.sqrt(2 * s.n_layer)
    for name, shp, _ in param_layout(s):
        n = int(np.prod(shp))
        if name.endswith("c_proj.weight"):
            a = rng.normal(0.0, resid_std, n)
        elif name in ("wte", "wpe") or name.endswith("attn.c_attn.weight") or name.endswith("mlp.c_fc.weight"):
            a = rng.normal(0.0, 0.02, n)
        elif ".ln_" in name or name.startswith("ln_f"):
            a = np.ones(n) if name.endswith("weight") else np.zeros(n)
        else:  # Linear biases
            a = np.zeros(n)
        chunks.append(a)
    return np.concatenate(chunks).astype(dtype)


def random_params(s: ModelShape, seed: int, scale: float = 0.02, dtype=np.float32) -> np.ndarray:
    """Every parameter (LN and biases included) drawn N(0, scale); LN weights around 1.

    Used by parity tests so that biases and LayerNorm affine terms are exercised
    with non-trivial values.
    """
    rng = np.random.default_rng(seed)
    chunks = []
    for name, shp, _ in param_layout(s):
        n = int(np.prod(shp))
        a = rng.normal(0.0, scale, n)
        if (".ln_" in name or name.startswith("ln_f")) and name.endswith("weight"):
            a = 1.0 + 5.0 * a
        chunks.append(a)
    return np.concatenate(chunks).astype(dtype)


def uniform_tokens(B: int, T: int, vocab: int, seed: int):
    """B rows of T+1 uniform ids; returns (idx, targets) int32, targets shifted by one."""
    rng = np.random.default_rng(seed)
    rows = rng.integers(0, vocab, size=(B, T + 1), dtype=np.int64)
    return rows[:, :T].astype(np.int32), rows[:, 1:].astype(np.int32)


def _zipf_cdf(vocab: int, s: float) -> np.ndarray:
    w = np.arange(1, vocab + 1, dtype=np.float64) ** (-s)
    c = np.cumsum(w)
    return c / c[-1]


def zipf_tokens(B: int, T: int, vocab: int, seed: int, s: float = 1.1, rng=None):
    """B rows of T+1 ids with P(id = k-1) proportional to k**-s, k = 1..vocab.

    Sampled by inverse CDF from a seeded PCG64 stream. Returns (idx, targets)
    as int32 arrays, targets being the same rows shifted by one position.
    """
    if rng is None:
        rng = np.random.default_rng(seed)
    u = rng.random((B, T + 1))
    rows = np.searchsorted(_zipf_cdf(vocab, s), u, side="right")
    rows = np.minimum(rows, vocab - 1)
    return rows[:, :T].astype(np.int32), rows[:, 1:].astype(np.int32)


def masked_prefix(targets: np.ndarray, rng, lo: float = 0.2, hi: float = 0.6) -> np.ndarray:
    """SFT-style loss masking: a contiguous prefix of floor(U[lo,hi] * T) targets per row set to -1."""
    out = targets.copy()
    B, T = out.shape
    u = rng.uniform(lo, hi, size=B)
    for b in range(B):
        out[b, : int(math.floor(u[b] * T))] = -1
    return out


def accumulation_batches(n_micro: int, B: int, T: int, vocab: int, seed: int):
    """The gradient-accumulation workload: n_micro Zipf micro-batches; the second
    half get masked target prefixes. Returns a list of (idx, targets)."""
    rng = np.random.default_rng(seed)
    out = []
    for k in range(n_micro):
        idx, tgt = zipf_tokens(B, T, vocab, seed, rng=rng)
        if k >= n_micro // 2:
            tgt = masked_prefix(tgt, rng)
        out.append((idx, tgt))
    return out


def uniforms(n_steps: int, B: int, seed: int) -> np.ndarray:
    """(n_steps, B) float32 uniforms in [0, 1) from default_rng(seed): the random
    numbers of the multinomial draws of generation, one per drawn token."""
    return np.random.default_rng(seed).random((n_steps, B)).astype(np.float32)
