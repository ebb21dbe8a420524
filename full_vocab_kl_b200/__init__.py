"""Full-vocabulary hidden-state distillation loss for B200 (sm_100a).

Student and teacher pass their final hidden states; the library rebuilds the logits
one vocabulary block at a time on tcgen05 tensor cores and accumulates the
generalized JSD with an online log-sum-exp, never materialising [tokens, V].
"""

from . import _abi  # noqa: F401
from .api import (  # noqa: F401
    IGNORE_INDEX,
    device_status,
    forward_kl,
    generalized_jsd,
    kl_backward,
    kl_forward,
    make_shape,
    reverse_kl,
    workspace_bytes,
)
