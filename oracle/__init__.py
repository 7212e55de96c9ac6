"""CPU oracle for Lizard hybrid attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (the CUDA library and its Python binding) never does.
"""

from .lizard_ref import (  # noqa: F401
    gate_log_decay,
    layer_log_decay,
    feature_map,
    feature_map_backward,
    gla_forward,
    gla_backward,
    swa_forward,
    swa_backward,
    lizard_forward,
    lizard_backward,
    lizard_decode_step,
    attention_mse,
    lizard_stage1_step,
    gla_segment_state,
    chain_states,
    BRANCH_BOTH,
    BRANCH_GLA_ONLY,
    BRANCH_SWA_ONLY,
    GATE_PER_DIM,
    GATE_SCALAR,
)
