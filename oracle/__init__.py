"""The oracle of the column-sparse delta method: plain fp64 CPU code, test infrastructure only.

Only the tests, the smoke check in ``__graft_entry__`` and the CPU-baseline /
reference legs of ``bench.py`` may import this package; the CUDA library never
does, and it shares no code with it.

The module-level functions are the C++ oracle (``chipmunk_oracle.cpp``, through
``cpp.CppOracle``; built with g++ on first use). ``numpy_oracle`` is an
independent numpy restatement of the same functions with the same signatures,
kept as a cross-check that the C++ oracle must match.
"""
from . import chipmunk_oracle as numpy_oracle
from .cpp import FUNCTIONS, NEG_INF, CppOracle, default  # noqa: F401


def _delegate(name):
    def fn(*args, **kwargs):
        return getattr(default(), name)(*args, **kwargs)
    fn.__name__ = name
    fn.__qualname__ = name
    fn.__doc__ = getattr(numpy_oracle, name).__doc__
    return fn


for _name in FUNCTIONS:
    globals()[_name] = _delegate(_name)
del _name
