"""B200-native LAGS sparsification: error feedback, layer-wise exact top-k,
deterministic sparse aggregation and the SGD update, as hand-written sm_100a
CUDA kernels behind the C ABI in include/lags.h.

Importing the package loads liblags.so and fails if it is missing; there is no
CPU fallback.
"""
from ._binding import (  # noqa: F401
    EXPORTED, LAGS_ERR_ALIGNMENT, LAGS_ERR_BAD_PICKS, LAGS_ERR_CUDA, LAGS_ERR_INTERNAL,
    LAGS_ERR_INVALID_ARG, LAGS_ERR_TIMEOUT, LAGS_ERR_UNSUPPORTED_DEVICE, LAGS_ERR_WORKSPACE,
    LAGS_ERR_WRONG_DEVICE, LAGS_FLAG_BAD_PICKS, LAGS_FLAG_INTERNAL, LAGS_FLAG_TIMEOUT,
    LAGS_MAX_ELEMENTS, LAGS_MAX_WORKERS, LAGS_OK, LAGS_STAGE_WAIT_POLLS, LIB_PATH, LagsError,
    lags_adaptive_densities, lags_aggregate, lags_aggregate_apply, lags_apply,
    lags_dense_finish, lags_dense_sum, lags_error_string, lags_merge_layers,
    lags_plan_aggregate_workspace_bytes, lags_plan_create, lags_plan_create_range,
    lags_plan_destroy, lags_plan_info, lags_plan_kernel_launches, lags_plan_layer,
    lags_plan_set_events, lags_plan_set_index_wait_limit, lags_plan_set_stage_wait_limit,
    lags_plan_set_workspace,
    lags_sparsify, lags_sparsify_static, lags_static_status_poll, lags_status_poll, library,
)


def __getattr__(name):
    if name == "Plan":
        from .plan import Plan
        return Plan
    if name == "DenseKernels":
        from .plan import DenseKernels
        return DenseKernels
    raise AttributeError(name)
