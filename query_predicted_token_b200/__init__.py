"""Predicted-query token-level sparse decode attention for B200 (sm_100a).

The compute path is the CUDA library ``libasp.so`` (C ABI in ``include/asp.h``);
this package only builds it and marshals arguments to it.
"""
from ._lib import (  # noqa: F401
    ASP_BF16,
    ASP_F32,
    ASP_DEV_BAD_INDEX,
    ASP_DEV_BAD_PAGE,
    ASP_DEV_NAN_SCORE,
    ASP_DEV_SELECT,
    ASP_DEV_TAIL_LIMIT,
    ASP_DEV_WAIT_LIMIT,
    AspError,
    append_kv,
    DecodeState,
    KV,
    PredCfg,
    attend_workspace_bytes,
    check_wait_limit,
    device_status,
    event_handle,
    lib,
    make_event,
    predict_query,
    quest_build_meta,
    quest_page_scores,
    quest_select,
    score_keys,
    score_keys_cuda_cores,
    select_topk,
    sparse_attend,
    status_string,
    wait_selection,
)
