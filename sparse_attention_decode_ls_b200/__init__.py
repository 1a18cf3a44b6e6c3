"""B200-native (sm_100a) sparse-attention decode: indexer -> top-k -> hot buffer /
miss gather -> sparse MLA attention, exported as the C ABI in include/ls.h and bound
here through ctypes (``binding``).  ``synthetic`` draws the seeded test/bench inputs."""
from . import binding, synthetic  # noqa: F401

__all__ = ["synthetic", "binding"]
