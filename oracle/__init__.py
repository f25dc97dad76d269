"""The SeedLM oracle: a plain, slow, obviously correct CPU definition of the
seed-decompress matmul path.  TEST INFRASTRUCTURE: only tests/, the smoke
check and bench.py's CPU-baseline leg may import it; the product never does."""
from .oracle import *  # noqa: F401,F403
from . import oracle as oracle  # noqa: F401
