"""DuoLM multi-item-scoring ranker on B200 (sm_100a).

The work is done by the CUDA library ``libduolm.so`` (C ABI in
``include/duolm.h``); ``shared_prefix_item_b200._lib`` only marshals
arguments to it.  The public names below load the library on first use and
fail loudly if it has not been built (``python -m
shared_prefix_item_b200.build``); importing the ``build`` submodule does not
load it.
"""
_PUBLIC = ("DTYPE_BF16", "DTYPE_FP32", "MODE_INDEPENDENT", "MODE_MIS", "DuolmError", "Ranker", "attention_plan",
           "compile_requests", "lib", "lib_path")


def __getattr__(name):
    if name in _PUBLIC:
        from . import _lib
        return getattr(_lib, name)
    raise AttributeError(name)


__all__ = list(_PUBLIC)
