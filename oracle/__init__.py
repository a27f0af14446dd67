"""CPU oracle for the NF4 + double-quantization weight path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product library (``quantized_linear_layers_nf4_b200``) never imports it and
shares no code with it.
"""
from .nf4_oracle import *  # noqa: F401,F403
