"""CPU oracle for the HATA decode step (test infrastructure only; see hata_oracle)."""
from .hata_oracle import *  # noqa: F401,F403
from .hata_oracle import __all__  # noqa: F401
