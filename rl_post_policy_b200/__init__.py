"""B200 (sm_100a) fused GRPO/BNPO policy loss: Python side of libpl.so.

The binding (``rl_post_policy_b200.binding``) is loaded on first attribute
access, so ``python -m rl_post_policy_b200.build`` can rebuild the library
without loading an older copy of it.  Accessing any entry point when libpl.so
has not been built raises ImportError: there is no fallback path.
"""
import importlib


def __getattr__(name):
    if name.startswith("__") or name in ("binding", "build"):
        raise AttributeError(name)
    return getattr(importlib.import_module(__name__ + ".binding"), name)
