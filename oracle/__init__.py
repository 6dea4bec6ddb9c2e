"""CPU oracle for the GigaAM Conformer encoder + CTC hot path.

TEST INFRASTRUCTURE ONLY.  This package is the slow, plain definition of what
the CUDA path computes.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import it; the product path
(``conformer_speech_recognition_b200``) never does, and the two share no code.

It is written in NumPy (fp64 by default; fp32 for the timed CPU baseline) from
the pages' descriptions, each function citing the passage it follows:
``gigaam`` holds the encoder and the CTC head, ``rnnt`` the RNNT head and its
greedy decoding.  Pins
(tests under ``tests/test_oracle_*.py``) tie it to facts the pages and the
mathematics fix.  Parity of the full layer composition beyond those pins is
"parity unpinned": no page prints tensors, so on synthetic weights the oracle
is the definition.
"""
from . import gigaam as _gigaam
from . import rnnt as _rnnt
from .gigaam import *  # noqa: F401,F403
from .rnnt import *  # noqa: F401,F403

__all__ = list(_gigaam.__all__) + list(_rnnt.__all__)
