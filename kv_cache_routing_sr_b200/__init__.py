"""B200-native SinkRouter single-token decode attention.

The compute path is the C-ABI library ``libsinkrouter.so`` (hand-written CUDA
for sm_100a, declared in ``include/sinkrouter.h``); ``native`` is its thin
ctypes binding. Importing this package does not load the library; the first
call into ``native`` does, and raises if it is missing or cannot run.
"""
from importlib import import_module

__all__ = ["native", "inputs", "multilayer", "context_parallel", "proxy_quality", "build"]


def __getattr__(name):
    if name in __all__:
        return import_module(f"{__name__}.{name}")
    raise AttributeError(name)
