"""B200 (sm_100a) block-sparse attention: BlockMask builders, fused forward,
decode against a KV cache, and backward.

The package exposes the C-ABI of libfa.so (include/fa.h) under the same names
(``fa_create_block_mask``, ``fa_flex_attention_fwd``, ``fa_flex_attention_bwd``,
...) plus thin torch conveniences (``create_block_mask``, ``flex_attention``,
``flex_attention_decode``, ``flex_attention_backward``, ...); see ``_binding``.

The library is loaded on first use of any of those names.  There is no
fallback: if libfa.so is missing, that first use raises ImportError.  Build the
library with ``python -m block_sparse_attention_create_b200.build`` (this
submodule does not need the library).
"""
import importlib

_SUBMODULES = ("build",)


def __getattr__(name):
    if name in _SUBMODULES:
        return importlib.import_module(f".{name}", __name__)
    if name.startswith("__"):
        raise AttributeError(name)
    binding = importlib.import_module("._binding", __name__)
    return getattr(binding, name)
