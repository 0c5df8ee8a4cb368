"""fp64 CPU oracle for the BaKron solver: test infrastructure, never the product path.

Only the tests, the smoke check and the CPU-baseline leg of the benchmark may import this
package. It shares no code with the CUDA library.
"""
from .bakron_oracle import *  # noqa: F401,F403
