"""CPU oracle for the Muon optimizer step and the AdamW step of the remaining
parameters (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path
(``newton_schulz_norm_b200``) never imports, links or executes it, and it
imports nothing from the product path.

Every function is a plain fp64 NumPy restatement of the step, with bf16
round-to-nearest-even applied at the storage points the GPU uses.  See
``oracle/muon_ref.py`` and ``oracle/adamw_ref.py`` for the passages each
function follows.
"""
from .muon_ref import (  # noqa: F401
    EPS,
    BF16_MAX,
    bf16_round,
    f32_round,
    coeffs_f32,
    momentum_ref,
    normalize_ref,
    orient,
    newton_schulz_ref,
    update_scale,
    muon_step_ref,
    orthogonalize_ref,
)
from .adamw_ref import (  # noqa: F401
    adamw_tensor_ref,
    adamw_update_term,
    adamw_step_ref,
    adamw_trajectory,
)
