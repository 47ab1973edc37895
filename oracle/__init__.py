"""CPU oracle of the NVFP4 linear-layer training path (test infrastructure).

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference legs
may import this package.  It never imports the CUDA library or the product
package, and the product never imports it.
"""
from .oracle import *  # noqa: F401,F403
