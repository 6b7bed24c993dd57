"""B200 (sm_100a) library for the chunked TTT-KVB fast-weight layer and its parallel
linear-attention form. ``abi`` is the thin binding of the C ABI (include/ttt.h);
``layer`` wraps it for torch tensors (allocation of outputs and workspace only)."""
from . import abi  # noqa: F401  (loads the shared library lazily, on first call)
