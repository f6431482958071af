"""Float64 CPU oracle of the H3-Omni block step (test infrastructure only).

Imported only by tests/, the graft smoke entry and the bench's CPU-baseline
leg; the CUDA library never imports, links or calls it.
"""
from . import h3_oracle, h3_loops  # noqa: F401
