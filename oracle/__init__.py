"""CPU oracle for the In-Place TTT fast-weight MLP forward.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, the smoke check and the
benchmark's CPU-baseline leg, never by the library.  See ``ittt_oracle.py``.
"""

from . import brute, ittt_oracle

__all__ = ["brute", "ittt_oracle"]
