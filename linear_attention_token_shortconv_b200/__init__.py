"""B200 (sm_100a) Gated DeltaNet token mixer: a C-ABI CUDA library and its binding.

``gdn.prefill`` / ``gdn.decode_step`` call the in-tree ``libgdn.so``; ``workloads``
draws the seeded synthetic inputs.
"""
from . import gdn, workloads  # noqa: F401
from .gdn import GdnError, decode_step, prefill, prefill_workspace_size  # noqa: F401
