"""CPU oracle for QSA decode (test infrastructure; never imported by the product path)."""
from . import qsa_oracle  # noqa: F401
