"""CPU oracle for the OasisKV lookahead sparse-KV decode path.

Test infrastructure only: imported by the tests, the smoke check and the
CPU-baseline leg of the benchmark, never by the product library.
"""
from .oasis_oracle import *  # noqa: F401,F403
from .oasis_oracle import default_scale  # noqa: F401
