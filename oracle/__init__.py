"""Oracle package -- TEST INFRASTRUCTURE ONLY (see oracle.armt)."""
from . import armt  # noqa: F401
