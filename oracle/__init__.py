"""Float64 CPU oracle for exact attention. Test infrastructure only.

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU baseline /
reference arm may import this package. The product path never uses it.
"""
from .ref import *  # noqa: F401,F403
from .ref import __all__  # noqa: F401
