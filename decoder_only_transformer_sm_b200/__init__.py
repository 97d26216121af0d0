"""B200-native GPT-2 training step: a C-ABI CUDA library (include/gpt2.h) and
its ctypes binding (``decoder_only_transformer_sm_b200.native``). Importing the
package does not load the library; constructing ``native.GPT2`` does, and
raises if it has not been built."""
from . import synthetic  # noqa: F401

__all__ = ["synthetic", "native"]
