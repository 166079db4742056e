"""Float64 CPU oracle for cross-model attention-map reuse.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package. The product path (the CUDA library and its Python
binding) never imports, links or calls it, and it never imports the product.
"""

from .iamap_oracle import *  # noqa: F401,F403
