"""S3R per-round hot path on B200: Python binding of libs3r.so (hand-written sm_100a kernels).

Importing this package loads the in-tree libs3r.so and fails loudly (ImportError) if it
has not been built; there is no fallback path.
"""
from ._lib import (  # noqa: F401
    BatchDesc,
    KVCacheDesc,
    MAX_K,
    PAGE_SIZE,
    S3RError,
    STATUS_NAMES,
    LIB_PATH,
    lib,
    make_batch,
    make_cache,
    new_workspace,
    s3r_choose_horizon,
    s3r_commit,
    s3r_sched_simulate,
    s3r_draft_argmax,
    s3r_draft_sample,
    s3r_draft_sample_noalloc,
    s3r_get_error,
    s3r_greedy_verify,
    s3r_horizon_step,
    s3r_launch_count,
    s3r_philox,
    s3r_position_scores,
    s3r_select_from_scores,
    s3r_select_kv_pages,
    s3r_select_pages_from_scores,
    s3r_select_kv,
    s3r_set_verify_kernel,
    s3r_set_wait_limit,
    s3r_sparse_draft_attn,
    s3r_spec_sample,
    s3r_status_string,
    s3r_verify_attn,
    s3r_workspace_init,
    s3r_workspace_size,
)
from .engine import AdaptiveHorizon, MixedPhaseDriver, RoundBuffers, S3REngine  # noqa: F401
