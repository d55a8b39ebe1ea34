"""B200-native speech front end and ASR encoder behind the ``libsal`` C-ABI.

``speech_audio_encoder_b200.api`` holds the thin Python binding (argument marshalling
over ctypes; every step runs in the CUDA library). ``speech_audio_encoder_b200.synth``
holds the seeded input generators. Importing the package loads nothing; the shared
library is loaded on first use and its absence is an error, never a fallback.
"""
__all__ = ["api", "synth"]
