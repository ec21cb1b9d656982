"""fp64 CPU oracle (test infrastructure only; see ``oracle.ref``)."""
from . import ref  # noqa: F401
