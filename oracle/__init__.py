"""Float64 CPU oracle (test infrastructure only; see ``sts_oracle``)."""

from .sts_oracle import (  # noqa: F401
    RowFilter,
    backward,
    entropy,
    filter_row,
    filter_rows,
    forward,
    logit_grad,
    logprob_on_prefix,
    policy_grad,
    row_gaps,
    sample_rows,
    scaled_logits,
)
