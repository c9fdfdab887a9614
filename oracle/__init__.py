"""CPU oracle for the NVFP4 SwiGLU FFN -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import this package.  The library (the CUDA path and its
binding) never imports, calls or links anything in here, and this package
never imports the library: the two share nothing but the seeded input
generator in ``nvfp4_quantized_dense_w4a16_b200.synth``, which draws random
numbers and holds none of the method's arithmetic.

Everything here is plain numpy, slow and written to be checked by eye against
the definitions it cites (see ``nvfp4_ffn``).
"""
from .nvfp4_ffn import *  # noqa: F401,F403
