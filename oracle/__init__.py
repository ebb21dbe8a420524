"""fp64 CPU oracle of the distillation loss — test infrastructure, never a product path.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs import this package.
"""

from .kl_oracle import (  # noqa: F401
    IGNORE_INDEX,
    backward,
    divergence_rows,
    dloss_du_student,
    forward,
    log_softmax,
    tempered_logits,
)
from . import spectral  # noqa: F401
