"""fp64 CPU oracle for exact attention -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs use this package.  It never imports the CUDA product
package and the product never imports it.
"""
from .attn_ref import *  # noqa: F401,F403
from .attn_ref import __all__  # noqa: F401
