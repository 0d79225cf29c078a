"""CPU oracle (float64) for the RG-LRU temporal core and Griffin's local attention.

Test infrastructure only: used by the test suite, the smoke check and the
benchmark's CPU-baseline leg, never by the product path."""
from .rglru_oracle import (  # noqa: F401
    C_DECAY, sigmoid, conv1d_causal, gate_preactivations, decay_direct, decay_log_space,
    rglru_recurrence, rglru_forward, ring_to_time_order, rglru_step, gelu,
    recurrent_block, RMS_EPS, rms_norm, gated_mlp, hawk_residual_layer,
    hawk_residual_layer_step, rglru_backward, max_rel_error,
)
from .local_attention import (  # noqa: F401
    ROPE_BASE, WINDOW, rope, local_mqa, local_attention, local_attention_step, griffin_attention_layer,
    griffin_attention_layer_step,
)
