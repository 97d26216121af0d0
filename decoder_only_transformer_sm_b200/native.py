"""ctypes binding of libgpt2_b200.so (include/gpt2.h): argument marshalling only.

Every step of the training step runs in the library's CUDA kernels; this module
only converts Python/torch/numpy arguments into the C ABI's pointers and sizes.
If the library is missing the calls raise: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgpt2_b200.so")

GPT2_OK = 0
ERRORS = {
    -1: "INVALID_ARG", -2: "OOM", -3: "CUDA", -4: "UNSUPPORTED_ARCH",
    -5: "NONFINITE", -6: "BAD_TOKEN", -7: "TIMEOUT",
}
PRECISION = {"fp32": 0, "bf16": 1}


class Gpt2Error(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"GPT2_ERR_{ERRORS.get(code, code)} ({code}): {msg}")
        self.code = code


class Config(ctypes.Structure):
    _fields_ = [
        ("n_layer", ctypes.c_int32), ("n_head", ctypes.c_int32), ("n_embd", ctypes.c_int32),
        ("vocab_size", ctypes.c_int32), ("block_size", ctypes.c_int32),
        ("max_B", ctypes.c_int32), ("max_T", ctypes.c_int32), ("precision", ctypes.c_int32),
        ("seed", ctypes.c_uint64), ("grad_clip", ctypes.c_float), ("flags", ctypes.c_uint32),
    ]


class KernelStat(ctypes.Structure):
    _fields_ = [
        ("name", ctypes.c_char * 96), ("launches", ctypes.c_int64), ("total_ms", ctypes.c_double),
        ("flops", ctypes.c_double), ("bytes", ctypes.c_double),
    ]


class TensorInfo(ctypes.Structure):
    _fields_ = [
        ("name", ctypes.c_char * 48), ("ndim", ctypes.c_int32), ("shape", ctypes.c_int64 * 2),
        ("offset", ctypes.c_int64), ("decay", ctypes.c_int32),
    ]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library once; raise if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} not found: build it with `python -m decoder_only_transformer_sm_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    sig = {
        "gpt2_last_error": (ctypes.c_char_p, []),
        "gpt2_create": (I, [ctypes.POINTER(Config), P, ctypes.POINTER(P)]),
        "gpt2_destroy": (None, [P]),
        "gpt2_set_stream": (I, [P, P]),
        "gpt2_num_params": (I, [P, ctypes.POINTER(ctypes.c_int64)]),
        "gpt2_param_layout": (I, [P, P, I, ctypes.POINTER(I)]),
        "gpt2_set_params": (I, [P, P, I]),
        "gpt2_get_params": (I, [P, P, I]),
        "gpt2_get_grads": (I, [P, P, I]),
        "gpt2_grads_device": (I, [P, ctypes.POINTER(P), ctypes.POINTER(ctypes.c_int64)]),
        "gpt2_debug_activation": (I, [P, I, I, I, I, P]),
        "gpt2_get_opt_state": (I, [P, P, P, ctypes.POINTER(ctypes.c_int64), I]),
        "gpt2_set_opt_state": (I, [P, P, P, ctypes.c_int64, I]),
        "gpt2_forward": (I, [P, P, P, I, I, P, ctypes.POINTER(F)]),
        "gpt2_forward_last": (I, [P, P, I, I, P]),
        "gpt2_prefill": (I, [P, P, I, I, P]),
        "gpt2_decode": (I, [P, P, I, I, P]),
        "gpt2_sample": (I, [P, P, I, F, I, P, P]),
        "gpt2_generate": (I, [P, P, I, I, I, F, I, P, P]),
        "gpt2_lr_at": (I, [ctypes.c_int64, F, F, ctypes.c_int64, ctypes.c_int64, ctypes.POINTER(F)]),
        "gpt2_zero_grad": (I, [P]),
        "gpt2_accumulate": (I, [P, P, P, I, I, F]),
        "gpt2_update": (I, [P, F, ctypes.POINTER(F), ctypes.POINTER(F)]),
        "gpt2_step": (I, [P, P, P, I, I, F, ctypes.POINTER(F), ctypes.POINTER(F)]),
        "gpt2_step_host": (I, [P, P, P, I, I, F, ctypes.POINTER(F), ctypes.POINTER(F)]),
        "gpt2_last_launch_count": (I, [P, ctypes.POINTER(ctypes.c_int64)]),
        "gpt2_grad_buckets": (I, [P, P, P, I, ctypes.POINTER(I)]),
        "gpt2_set_grad_events": (I, [P, P, I]),
        "gpt2_profile": (I, [P, I]),
        "gpt2_profile_read": (I, [P, P, I, ctypes.POINTER(I)]),
        "gpt2k_matmul_bf16": (I, [I, P, P, I, I, I, I, P, ctypes.c_int64, P, P, P, P, P, F, I, P, P]),
        "gpt2k_attention_fwd": (I, [I, P, P, P, I, I, I, I, I, P, P]),
        "gpt2k_attention_bwd": (I, [I, P, P, P, P, P, I, I, I, I, P, P, I, P, P]),
        "gpt2k_attention_bwd_workspace": (I, [I, I, I, I, I, ctypes.POINTER(ctypes.c_int64)]),
        "gpt2k_attention_decode": (I, [I, P, P, I, I, I, I, I, P, P, P]),
        "gpt2k_sample": (I, [I, P, I, I, ctypes.c_int64, F, I, P, P, P, P]),
        "gpt2k_embedding_bwd": (I, [P, P, I, I, I, I, P, P, P, P, P]),
        "gpt2k_embedding_bwd_workspace": (I, [I, I, I, ctypes.POINTER(ctypes.c_int64)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _check(rc: int):
    if rc != GPT2_OK:
        raise Gpt2Error(rc, load_library().gpt2_last_error().decode())


def _ptr(x) -> int | None:
    """Raw address of a torch tensor or numpy array (None passes NULL)."""
    if x is None:
        return None
    if isinstance(x, np.ndarray):
        assert x.flags["C_CONTIGUOUS"]
        return x.ctypes.data
    assert x.is_contiguous()
    return x.data_ptr()


class _DeviceArray:
    """A device float32 vector the library owns, described by the CUDA array
    interface so that torch.as_tensor can wrap it without a copy."""

    def __init__(self, ptr: int, n: int):
        self.__cuda_array_interface__ = {"shape": (n,), "typestr": "<f4", "data": (ptr, False), "version": 3,
                                         "strides": None}


class GPT2:
    """One model on the current CUDA device, created through gpt2_create."""

    def __init__(self, n_layer: int, n_head: int, n_embd: int, vocab_size: int, block_size: int,
                 max_B: int, max_T: int, precision: str = "bf16", seed: int = 0, grad_clip: float = 1.0,
                 stream=None):
        lib = load_library()
        self._lib = lib
        cfg = Config(n_layer, n_head, n_embd, vocab_size, block_size, max_B, max_T,
                     PRECISION[precision], seed, grad_clip, 0)
        h = ctypes.c_void_p()
        _check(lib.gpt2_create(ctypes.byref(cfg), stream, ctypes.byref(h)))
        self._h = h
        self.cfg = cfg
        self.precision = precision
        n = ctypes.c_int64()
        _check(lib.gpt2_num_params(h, ctypes.byref(n)))
        self.n_params = n.value

    def close(self):
        if getattr(self, "_h", None):
            self._lib.gpt2_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_stream(self, stream_ptr):
        _check(self._lib.gpt2_set_stream(self._h, stream_ptr))

    def layout(self):
        cnt = ctypes.c_int()
        _check(self._lib.gpt2_param_layout(self._h, None, 0, ctypes.byref(cnt)))
        arr = (TensorInfo * cnt.value)()
        _check(self._lib.gpt2_param_layout(self._h, arr, cnt.value, ctypes.byref(cnt)))
        out = []
        for t in arr:
            shape = tuple(int(t.shape[i]) for i in range(t.ndim))
            out.append((t.name.decode(), shape, int(t.offset), bool(t.decay)))
        return out

    # ---- flat state (host numpy float32 or device torch float32) ----
    def set_params(self, flat):
        on_dev = 0 if isinstance(flat, np.ndarray) else 1
        if on_dev == 0:
            flat = np.ascontiguousarray(flat, dtype=np.float32)
        assert flat.size == self.n_params if on_dev == 0 else flat.numel() == self.n_params
        _check(self._lib.gpt2_set_params(self._h, _ptr(flat), on_dev))

    def get_params(self) -> np.ndarray:
        out = np.empty(self.n_params, np.float32)
        _check(self._lib.gpt2_get_params(self._h, _ptr(out), 0))
        return out

    def get_grads(self) -> np.ndarray:
        out = np.empty(self.n_params, np.float32)
        _check(self._lib.gpt2_get_grads(self._h, _ptr(out), 0))
        return out

    ACT = {"resid": 0, "ln_1": 1, "qkv": 2, "attn": 3, "ln_2": 4, "gelu": 5, "ln_f": 6}

    def debug_activation(self, kind: str, index: int, B: int, T: int) -> np.ndarray:
        """gpt2_debug_activation: a saved activation of the last forward as float32 (B, T, width)."""
        width = {"qkv": 3, "gelu": 4}.get(kind, 1) * self.cfg.n_embd
        out = np.empty((B, T, width), np.float32)
        _check(self._lib.gpt2_debug_activation(self._h, self.ACT[kind], index, B, T, _ptr(out)))
        return out

    def grads_view(self):
        """The handle's gradient vector as a torch float32 CUDA tensor sharing its
        memory (gpt2_grads_device; no copy), for in-place collectives."""
        import torch
        ptr, n = ctypes.c_void_p(), ctypes.c_int64()
        _check(self._lib.gpt2_grads_device(self._h, ctypes.byref(ptr), ctypes.byref(n)))
        return torch.as_tensor(_DeviceArray(ptr.value, n.value), device="cuda")

    def grad_buckets(self):
        """[(offset, count)] ranges of the flat gradient vector in the order the
        backward finishes them (gpt2_grad_buckets)."""
        n = ctypes.c_int()
        _check(self._lib.gpt2_grad_buckets(self._h, None, None, 0, ctypes.byref(n)))
        off = np.empty(n.value, np.int64)
        cnt = np.empty(n.value, np.int64)
        _check(self._lib.gpt2_grad_buckets(self._h, _ptr(off), _ptr(cnt), n.value, ctypes.byref(n)))
        return [(int(o), int(c)) for o, c in zip(off, cnt)]

    def set_grad_events(self, events):
        """torch.cuda.Event per bucket, recorded by every eager backward as each bucket
        becomes final (gpt2_set_grad_events); None stops the recording. The events are
        kept alive here while set."""
        if events is None:
            _check(self._lib.gpt2_set_grad_events(self._h, None, 0))
            self._grad_events = None
            return
        handles = (ctypes.c_void_p * len(events))(*[ev.cuda_event for ev in events])
        _check(self._lib.gpt2_set_grad_events(self._h, handles, len(events)))
        self._grad_events = list(events)

    def get_opt_state(self):
        m = np.empty(self.n_params, np.float32)
        v = np.empty(self.n_params, np.float32)
        t = ctypes.c_int64()
        _check(self._lib.gpt2_get_opt_state(self._h, _ptr(m), _ptr(v), ctypes.byref(t), 0))
        return m, v, t.value

    def set_opt_state(self, m, v, step: int):
        m = np.ascontiguousarray(m, np.float32)
        v = np.ascontiguousarray(v, np.float32)
        _check(self._lib.gpt2_set_opt_state(self._h, _ptr(m), _ptr(v), step, 0))

    # ---- compute (device int32 token tensors) ----
    def forward(self, idx, targets=None, logits=None):
        B, T = idx.shape
        loss = ctypes.c_float()
        _check(self._lib.gpt2_forward(self._h, _ptr(idx), _ptr(targets), B, T, _ptr(logits),
                                      ctypes.byref(loss) if targets is not None else None))
        return loss.value if targets is not None else None

    def forward_last(self, idx, logits):
        """Logits (B, vocab_size) of each sequence's last position (gpt2_forward_last)."""
        B, T = idx.shape
        _check(self._lib.gpt2_forward_last(self._h, _ptr(idx), B, T, _ptr(logits)))

    # ---- generation (device tensors; "A generation loop") ----
    def prefill(self, idx, logits):
        """gpt2_prefill: last-position logits (B, vocab_size) and the k/v cache of idx (B, T)."""
        B, T = idx.shape
        _check(self._lib.gpt2_prefill(self._h, _ptr(idx), B, T, _ptr(logits)))

    def decode(self, tokens, pos: int, logits):
        """gpt2_decode: tokens (B,) at position pos against the cache; logits (B, vocab_size)."""
        _check(self._lib.gpt2_decode(self._h, _ptr(tokens), tokens.shape[0], pos, _ptr(logits)))

    def sample(self, logits, temperature: float, top_k: int, u, next_tokens):
        """gpt2_sample: one draw per row of logits (B, vocab_size) at the uniforms u (B,)."""
        _check(self._lib.gpt2_sample(self._h, _ptr(logits), logits.shape[0], temperature, top_k, _ptr(u),
                                     _ptr(next_tokens)))

    def generate(self, prompt, max_new_tokens: int, temperature: float, top_k: int, u, out):
        """gpt2_generate: out (B, T0 + max_new_tokens) = prompt (B, T0) + drawn tokens; u (max_new_tokens, B)."""
        B, T0 = prompt.shape
        _check(self._lib.gpt2_generate(self._h, _ptr(prompt), B, T0, max_new_tokens, temperature, top_k, _ptr(u),
                                       _ptr(out)))

    def zero_grad(self):
        _check(self._lib.gpt2_zero_grad(self._h))

    def accumulate(self, idx, targets, loss_scale: float):
        B, T = idx.shape
        _check(self._lib.gpt2_accumulate(self._h, _ptr(idx), _ptr(targets), B, T, loss_scale))

    def update(self, lr: float):
        loss, norm = ctypes.c_float(), ctypes.c_float()
        _check(self._lib.gpt2_update(self._h, lr, ctypes.byref(loss), ctypes.byref(norm)))
        return loss.value, norm.value

    def step(self, idx, targets, lr: float):
        B, T = idx.shape
        loss, norm = ctypes.c_float(), ctypes.c_float()
        _check(self._lib.gpt2_step(self._h, _ptr(idx), _ptr(targets), B, T, lr,
                                   ctypes.byref(loss), ctypes.byref(norm)))
        return loss.value, norm.value

    def step_host(self, idx, targets, lr: float):
        """idx/targets: host int32 arrays or pinned CPU torch tensors."""
        B, T = idx.shape
        loss, norm = ctypes.c_float(), ctypes.c_float()
        _check(self._lib.gpt2_step_host(self._h, _ptr(idx), _ptr(targets), B, T, lr,
                                        ctypes.byref(loss), ctypes.byref(norm)))
        return loss.value, norm.value

    def profile(self, enable: bool = True):
        _check(self._lib.gpt2_profile(self._h, 1 if enable else 0))

    def profile_read(self):
        """List of dicts: name, launches, total_ms, flops, bytes (per launch site)."""
        cnt = ctypes.c_int()
        _check(self._lib.gpt2_profile_read(self._h, None, 0, ctypes.byref(cnt)))
        arr = (KernelStat * max(cnt.value, 1))()
        _check(self._lib.gpt2_profile_read(self._h, arr, cnt.value, ctypes.byref(cnt)))
        return [dict(name=a.name.decode(), launches=int(a.launches), total_ms=float(a.total_ms),
                     flops=float(a.flops), bytes=float(a.bytes)) for a in arr[:cnt.value]]

    def last_launch_count(self) -> int:
        n = ctypes.c_int64()
        _check(self._lib.gpt2_last_launch_count(self._h, ctypes.byref(n)))
        return n.value


# ---------------------------------------------------------------------------
# Kernel-level entry points (include/gpt2_kernels.h).
# ---------------------------------------------------------------------------
LAYOUT = {"NT": 0, "NN": 1, "TN": 2}
EPILOGUE = {"store": 0, "bias": 1, "bias_gelu": 2, "bias_resid": 3, "mul": 4, "accum_f32": 5}


def matmul_bf16(layout: str, A, B, M: int, N: int, K: int, epilogue: str, out, ldo: int | None = None,
                out2=None, bias=None, resid=None, aux=None, beta: float = 0.0, engine: str = "tc",
                status=None, stream=None, colsum_part=None):
    """gpt2k_matmul_bf16 on torch device tensors; returns the device status tensor."""
    import torch
    lib = load_library()
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=out.device)
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    rc = lib.gpt2k_matmul_bf16(LAYOUT[layout], _ptr(A), _ptr(B), M, N, K, EPILOGUE[epilogue], _ptr(out),
                               ldo if ldo is not None else N, _ptr(out2), _ptr(bias), _ptr(resid), _ptr(aux),
                               _ptr(colsum_part), beta, 1 if engine == "tc" else 0, _ptr(status), stream)
    _check(rc)
    return status


def lr_at(step: int, max_lr: float, min_lr: float, warmup: int, max_steps: int) -> float:
    """gpt2_lr_at: the warmup + cosine learning-rate schedule (host only, no GPU)."""
    out = ctypes.c_float()
    _check(load_library().gpt2_lr_at(step, max_lr, min_lr, warmup, max_steps, ctypes.byref(out)))
    return out.value


def _dtype_code(t) -> int:
    import torch
    return {torch.float32: 0, torch.bfloat16: 1}[t.dtype]


def _stream_and_status(ref, status, stream):
    import torch
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=ref.device)
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    return status, stream


def attention_fwd(qkv, out, lse, B: int, T: int, H: int, hd: int, engine: int = 0, status=None, stream=None):
    """gpt2k_attention_fwd on torch device tensors; returns the status tensor."""
    status, stream = _stream_and_status(qkv, status, stream)
    _check(load_library().gpt2k_attention_fwd(_dtype_code(qkv), _ptr(qkv), _ptr(out), _ptr(lse), B, T, H, hd,
                                              engine, _ptr(status), stream))
    return status


def attention_bwd_workspace(B: int, T: int, H: int, hd: int, engine: int = 0) -> int:
    """Float32 elements of the workspace gpt2k_attention_bwd needs (gpt2k_attention_bwd_workspace)."""
    n = ctypes.c_int64()
    _check(load_library().gpt2k_attention_bwd_workspace(B, T, H, hd, engine, ctypes.byref(n)))
    return n.value


def attention_bwd(qkv, out, dout, lse, dqkv, B: int, T: int, H: int, hd: int, workspace, engine: int = 0,
                  status=None, stream=None, colsum_part=None):
    """gpt2k_attention_bwd on torch device tensors (workspace: attention_bwd_workspace(...) float32)."""
    status, stream = _stream_and_status(qkv, status, stream)
    _check(load_library().gpt2k_attention_bwd(_dtype_code(qkv), _ptr(qkv), _ptr(out), _ptr(dout), _ptr(lse),
                                              _ptr(dqkv), B, T, H, hd, _ptr(workspace), _ptr(colsum_part), engine,
                                              _ptr(status), stream))
    return status


def attention_bwd_noalloc(qkv, out, dout, lse, dqkv, B: int, T: int, H: int, hd: int, engine: int = 0,
                          status=None, stream=None):
    """gpt2k_attention_bwd_noalloc: the attention backward with the library's own
    fixed scratch (B*H*T <= 262144), for callers that cannot allocate device memory."""
    lib = load_library()
    fn = lib.gpt2k_attention_bwd_noalloc
    if fn.argtypes is None:
        P, I = ctypes.c_void_p, ctypes.c_int
        fn.restype = I
        fn.argtypes = [I, P, P, P, P, P, I, I, I, I, I, P, P]
    status, stream = _stream_and_status(qkv, status, stream)
    _check(fn(_dtype_code(qkv), _ptr(qkv), _ptr(out), _ptr(dout), _ptr(lse), _ptr(dqkv), B, T, H, hd, engine,
              _ptr(status), stream))
    return status


def embedding_bwd_workspace(B: int, T: int, C: int) -> int:
    """Float32 elements of the workspace gpt2k_embedding_bwd needs."""
    n = ctypes.c_int64()
    _check(load_library().gpt2k_embedding_bwd_workspace(B, T, C, ctypes.byref(n)))
    return n.value


def embedding_bwd(idx, dx, dwte, dwpe, B: int, T: int, workspace=None, status=None, stream=None):
    """gpt2k_embedding_bwd: dwte[idx] += dx rows and dwpe[t] += sum over b, on torch
    device tensors (idx int32 (B*T), dx float32 (B*T, C), dwte (V, C), dwpe (T, C));
    with a workspace (embedding_bwd_workspace(...) float32) in a fixed order."""
    status, stream = _stream_and_status(dx, status, stream)
    _check(load_library().gpt2k_embedding_bwd(_ptr(idx), _ptr(dx), B, T, dx.shape[-1], dwte.shape[0], _ptr(dwte),
                                              _ptr(dwpe), _ptr(workspace), _ptr(status), stream))
    return status


def attention_decode(cache, out, B: int, H: int, hd: int, Tc: int, n: int, workspace, status=None, stream=None):
    """gpt2k_attention_decode: the newest position n-1 of each sequence against cache
    (B, Tc, 3C); workspace: B*H*ceil(Tc/64)*(hd+2) float32."""
    status, stream = _stream_and_status(cache, status, stream)
    _check(load_library().gpt2k_attention_decode(_dtype_code(cache), _ptr(cache), _ptr(out), B, H, hd, Tc, n,
                                                 _ptr(workspace), _ptr(status), stream))
    return status


def sample(logits, V: int, temperature: float, top_k: int, u, next_tokens, ld: int | None = None, status=None,
           stream=None):
    """gpt2k_sample on rows of logits (rows, ld) (first V columns); next_tokens (rows,) int32."""
    status, stream = _stream_and_status(logits, status, stream)
    rows = logits.shape[0]
    _check(load_library().gpt2k_sample(_dtype_code(logits), _ptr(logits), rows, V, ld if ld is not None else V,
                                       temperature, top_k, _ptr(u), _ptr(next_tokens), _ptr(status), stream))
    return status
