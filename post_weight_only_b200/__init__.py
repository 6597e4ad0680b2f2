"""B200-native AWQ per-layer activation-aware scale search.

The computation lives in the CUDA library ``libawq_b200.so`` (C ABI declared in
``include/awq_b200.h``); :mod:`post_weight_only_b200.awq` is its thin binding.
:mod:`post_weight_only_b200.synth` draws the seeded synthetic layers.
"""


def __getattr__(name):
    # Load the CUDA binding only when it is used, so that importing the
    # synthetic-input module does not require the built library.
    if name == "awq":
        import importlib
        return importlib.import_module(".awq", __name__)
    raise AttributeError(name)
