"""Float64 CPU oracle for the bidirectional Video Delta Attention branch.

Test infrastructure only: imported by tests/, by the smoke check and by the
CPU-baseline leg of bench.py, never by the product path.
"""
from .vda_ref import (  # noqa: F401
    RMS_EPS,
    batch_rule_update,
    decayed,
    boundary_states,
    boundary_states_by_chunk_maps,
    compose_maps,
    frame_map,
    frame_stats,
    frame_update,
    forward_scan,
    reverse_scan,
    gathered_state,
    gathered_state_frame,
    num_chunks,
    rms_gate,
    text_state,
    vda_forward,
    vda_forward_head,
    vda_forward_head_naive,
    window_bounds,
)
from .prep_ref import (  # noqa: F401
    L2_EPS,
    conv_spatial,
    conv_temporal,
    l2_normalize,
    prep,
    prep_head,
    short_conv,
    silu,
)
