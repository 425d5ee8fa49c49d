"""B200-native forward Differential Attention V2 (prefill and decode) behind a C ABI.

The CUDA library (libdiffattn_v2.so, sm_100a) does all the work; this package is its thin
ctypes binding. Build the library with `python -m differential_attention_v2_b200.build`.
The binding is loaded on first use of any of its names; if the library is missing that
use raises ImportError (there is no fallback implementation).
"""
import importlib

_BINDING_NAMES = (
    "prefill", "prefill_window", "prefill_varlen", "prefill_varlen_window", "prefill_f32", "prefill_train", "backward",
    "backward_workspace_size", "prefill_varlen_train", "backward_varlen", "backward_varlen_workspace_size", "decode", "decode_f32", "decode_workspace_size", "decode_noalloc", "decode_paged",
    "decode_multi", "lambda_v1", "lambda_v2", "prefill_fused_lambda", "device_error", "version", "load", "DiffAttnError", "EXPORTED", "LIB_PATH",
    "LIB",
)
__all__ = list(_BINDING_NAMES)


def __getattr__(name):
    if name in _BINDING_NAMES:
        mod = importlib.import_module("._lib", __name__)
        return getattr(mod, name)
    raise AttributeError(name)
