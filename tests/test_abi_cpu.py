"""Host-side checks of the C ABI (no GPU): the library loads, exports every
function include/*.h declares, and rejects bad configurations before touching
the device."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

from decoder_only_transformer_sm_b200 import native

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^[A-Za-z_][\w\s\*]*?\b(gpt2\w*)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    lib = native.load_library()
    decl = _declared_functions()
    assert len(decl) >= 18, decl
    out = subprocess.run(["nm", "-D", "--defined-only", native.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(\w+)$", out, flags=re.M))
    missing = [d for d in decl if d not in exported]
    assert not missing, missing
    for d in decl:
        getattr(lib, d)


def test_library_has_no_runtime_dependency_on_libcuda():
    out = subprocess.run(["ldd", native.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out and "libcudart.so" not in out


def _create(**kw):
    lib = native.load_library()
    base = dict(n_layer=2, n_head=4, n_embd=128, vocab_size=1024, block_size=64, max_B=4, max_T=64,
                precision=0, seed=0, grad_clip=1.0, flags=0)
    base.update(kw)
    cfg = native.Config(*[base[f] for f, _ in native.Config._fields_])
    h = ctypes.c_void_p()
    rc = lib.gpt2_create(ctypes.byref(cfg), None, ctypes.byref(h))
    return rc, lib.gpt2_last_error().decode(), h


@pytest.mark.parametrize("kw,msg", [
    (dict(n_head=3), "multiple of n_head"),
    (dict(n_embd=192, n_head=2), "32 or 64"),
    (dict(n_embd=96, n_head=3), "multiple of 64"),
    (dict(vocab_size=50257), "multiple of 8"),
    (dict(max_T=65), "block_size"),
    (dict(precision=7), "precision"),
    (dict(n_layer=0), ">= 1"),
    (dict(flags=1), "flags"),
])
def test_invalid_configs_rejected_on_host(kw, msg):
    rc, err, h = _create(**kw)
    assert rc == -1 and msg in err and not h.value


def test_null_arguments():
    lib = native.load_library()
    assert lib.gpt2_create(None, None, None) == -1
    h = ctypes.c_void_p()
    assert lib.gpt2_create(None, None, ctypes.byref(h)) == -1
    lib.gpt2_destroy(None)   # no-op
    n = ctypes.c_int64()
    assert lib.gpt2_num_params(None, ctypes.byref(n)) == -1


def test_lr_schedule_entry_matches_oracle():
    """gpt2_lr_at (host only: runs without a GPU) against the oracle's schedule,
    float32 rounding apart, over the 124M run's steps; bad arguments rejected."""
    from decoder_only_transformer_sm_b200 import native
    from oracle import gpt2_oracle as O
    mx, mn, tw, tm = 6e-4, 6e-5, 715, 19073
    for k in list(range(0, 800, 7)) + list(range(700, 19200, 211)) + [tw - 1, tw, tm, tm + 1, 50000]:
        assert native.lr_at(k, mx, mn, tw, tm) == pytest.approx(O.lr_schedule(k, mx, mn, tw, tm), rel=1e-6)
    for bad in [(-1, mx, mn, tw, tm), (0, mx, mn, 0, tm), (0, mx, mn, tw, tw - 1)]:
        with pytest.raises(native.Gpt2Error):
            native.lr_at(*bad)


def test_generation_entries_reject_bad_arguments_on_host():
    """The generation entry points validate their arguments before any CUDA
    call (no GPU needed): NULL handles and pointers, bad sizes, a temperature
    that is not finite and > 0, a row stride below V, n outside [1, Tc]."""
    lib = native.load_library()
    dummy = ctypes.c_void_p(16)   # never dereferenced: validation fails first
    assert lib.gpt2_prefill(None, dummy, 1, 1, dummy) == -1
    assert lib.gpt2_decode(None, dummy, 1, 1, dummy) == -1
    assert lib.gpt2_sample(None, dummy, 1, 1.0, 0, dummy, dummy) == -1
    assert lib.gpt2_generate(None, dummy, 1, 1, 1, 1.0, 0, dummy, dummy) == -1
    assert lib.gpt2_debug_activation(None, 0, 0, 1, 1, dummy) == -1
    assert lib.gpt2_grads_device(None, ctypes.byref(ctypes.c_void_p()), ctypes.byref(ctypes.c_int64())) == -1
    ok = (1, dummy, 4, 8, 8, 1.0, 0, dummy, dummy, dummy, None)
    for i, bad in [(0, 7), (2, 0), (3, 0), (4, 7), (5, 0.0), (5, float("nan")), (5, float("inf")), (7, None)]:
        args = list(ok)
        args[i] = bad
        assert lib.gpt2k_sample(*args) == -1, (i, bad)
    okd = (1, dummy, dummy, 2, 4, 64, 100, 100, dummy, dummy, None)
    for i, bad in [(0, 3), (3, 0), (5, 48), (6, 0), (7, 0), (7, 101), (8, None)]:
        args = list(okd)
        args[i] = bad
        assert lib.gpt2k_attention_decode(*args) == -1, (i, bad)


def test_embedding_bwd_rejects_bad_arguments_on_host():
    """gpt2k_embedding_bwd validates sizes and pointers before any CUDA call (no GPU
    needed): sizes below 1, C not a multiple of 4, NULL operands (the workspace
    alone may be NULL). Its workspace size is rows x C + rows + 64 floats."""
    lib = native.load_library()
    dummy = ctypes.c_void_p(16)   # never dereferenced: validation fails first
    ok = (dummy, dummy, 2, 4, 8, 100, dummy, dummy, None, dummy, None)
    for i, bad in [(2, 0), (3, 0), (4, 0), (4, 6), (5, 0), (0, None), (1, None), (6, None), (7, None), (9, None)]:
        args = list(ok)
        args[i] = bad
        assert lib.gpt2k_embedding_bwd(*args) == -1, (i, bad)
    n = ctypes.c_int64()
    assert lib.gpt2k_embedding_bwd_workspace(2, 4, 8, ctypes.byref(n)) == 0
    assert n.value == 8 * 8 + 8 + 64
    assert lib.gpt2k_embedding_bwd_workspace(0, 4, 8, ctypes.byref(n)) == -1
    assert lib.gpt2k_embedding_bwd_workspace(2, 4, 8, None) == -1
