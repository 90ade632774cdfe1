"""CPU oracle for the SA compression step (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package.  It shares no code with the CUDA
library and never calls it.
"""

from .sa_oracle import (  # noqa: F401
    DEFAULT_STEPS,
    affinity,
    aggregate,
    mass_normalised,
    project_keys,
    project_prototypes,
    prototype_mass,
    prototype_softmax,
    sa_batch,
    sa_batch_user_queries,
    sa_user,
)
from .brute import sa_user_bruteforce  # noqa: F401
from .sa_backward import sa_batch_backward, sa_user_backward  # noqa: F401
from .sa_refine import (  # noqa: F401
    layer_norm,
    refine_layer,
    refine_stack,
    refine_update,
    silu,
    swiglu_ffn,
)
from .sa_action import action_fuse, fusion_hidden, fusion_input  # noqa: F401
