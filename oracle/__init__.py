"""fp64 CPU oracle for the speech front end and ASR encoder (test infrastructure).

This package is test infrastructure, not product code. Only the test suite,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs of
``bench.py`` may import it. Its arithmetic is the plain C++ of ``sal_oracle.cpp``
(``liboracle.so``), reached through ``oracle.py``. It shares no code, tables or constants
generators with the CUDA library in ``speech_audio_encoder_b200``; the two meet only
through the seeded inputs of ``speech_audio_encoder_b200.synth``.
"""
from .oracle import *  # noqa: F401,F403
from .oracle import build  # noqa: F401
