"""CPU oracle for block-sparse causal prefill attention (FlashPrefill style).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline/reference leg may import it; the product path never does, and it
shares no code with the CUDA path.

Pinned by ``tests/test_oracle_pins.py`` (closed forms, library special cases,
brute force on tiny inputs, hand-derived fixtures under ``tests/golden``).
The V2 mean-correction term is undefined on the pages and is not implemented
(parity unpinned / excluded).
"""
from .flashprefill_oracle import *  # noqa: F401,F403
from .flashprefill_oracle import default_scale  # noqa: F401
from .brute_force import brute_force  # noqa: F401
