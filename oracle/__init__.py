"""CPU oracle for the LAGS sparsify / aggregate / apply path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this package.  The
product path (``layer_wise_top_b200``) never imports it and has no CPU
fallback.
"""
from .lags_oracle import (  # noqa: F401
    adaptive_densities, aggregate, aggregate_layer, apply_update, dense_sgd_update, error_feedback,
    k_of, layer_plan,
    magnitude_order, merge_layers, message_schedule_end, run_workload, select_layer, sparsify,
    sparsify_layer,
)
