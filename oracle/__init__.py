"""Oracle of the wave-index path (test infrastructure only; see wave_index)."""
from .wave_index import *  # noqa: F401,F403
from . import wave_index  # noqa: F401
