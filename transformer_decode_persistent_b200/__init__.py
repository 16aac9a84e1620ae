"""B200-native batch-1 decode engine: a persistent decode kernel behind a C ABI.

The library (``libkie.so``, built in-tree from ``csrc/``) exposes
kie_create / kie_load_weights / kie_prefill / kie_decode / kie_reset /
kie_destroy (see ``include/kie.h``); ``kie.Engine`` is the Python binding.
"""
from .kie import EXPORTS, Engine, KieError, lib  # noqa: F401
