"""CPU oracle for the ARL2 hybrid attention layer (test infrastructure only).

This package is the plain, slow, float64 statement of what the layer computes.
It exists to check the CUDA library, and nothing on the product path may use it:
only the test suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` import it.  It shares no code, tables
or helpers with ``gated_delta_linear_b200``, and neither side imports the other.

Source: "Technical summary: Attend Locally, Remember Linearly (ARL2)"
(gist.science/ar/paper/2605.16579), §2.1 "hybrid attention decomposition"
and §2.2 "memory-state management"; §1 for the key/value-cache softmax
baseline (``kvcache_attention``).  ``oracle.tra``: Token Radius Attention
("Technical summary: Token Radius Attention", gist.science/ar/paper/2608.02504)
on the intra-frame branch.
"""

from .hybrid_layer import (  # noqa: F401
    sigmoid,
    feature_map,
    l2_normalise_rows,
    intra_frame_attention,
    inter_frame_read,
    frame_gates,
    gated_delta_update,
    head_pass,
    layer_pass,
    run_frames,
    kvcache_attention,
    mixed_output,
    token_level_head_pass,
)
from . import tra  # noqa: F401
