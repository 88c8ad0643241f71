"""B200-native forward pass of the LinGen MATE block (CUDA library libmate + a thin Python binding).

The compute lives in libmate.so (built in-tree for sm_100a by `build.py`); `mate.py` marshals torch
tensors into the C ABI declared in include/mate.h.
"""
from . import _lib  # noqa: F401  (ctypes declarations; loads nothing until first use)


def __getattr__(name):
    # Import the torch-facing binding lazily so that `import linear_complexity_video_mate_b200` stays cheap.
    if name in ("mate",):
        import importlib
        return importlib.import_module(".mate", __name__)
    raise AttributeError(name)
