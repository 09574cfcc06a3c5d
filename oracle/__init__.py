"""fp64 CPU oracle of the hierarchical local attention layer.

Test infrastructure: only the tests, the smoke check and the benchmark's CPU
baseline import it.  It never imports the CUDA package, and the CUDA package
never imports it.
"""
from .hier_local_attn import *  # noqa: F401,F403
from .hier_local_attn import Geometry  # noqa: F401
