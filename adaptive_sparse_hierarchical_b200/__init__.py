"""B200-native DashAttention forward pass (Stage 0 summaries, Stage 1 entmax routing with the
GQA average, Stage 2 biased sparse softmax) behind the C ABI of include/dash.h."""
from ._lib import (DASH_BF16, DASH_F32, DASH_OP_DECODE, DASH_OP_PREFILL, DashError, dash_decode,
                   dash_decode_paged, dash_prefill, dash_prefill_stage, dash_route_capacity, dash_status_string,
                   dash_summary_append, dash_summary_append_paged, dash_summary_build, dash_summary_build_paged,
                   dash_workspace_size, load, paged_kv, params, route_out)
from .api import DecodeState, PagedDecodeState, Prefill, prefill

__all__ = ["DASH_BF16", "DASH_F32", "DASH_OP_DECODE", "DASH_OP_PREFILL", "DashError", "dash_decode",
           "dash_prefill", "dash_prefill_stage", "dash_route_capacity", "dash_status_string", "dash_summary_append",
           "dash_summary_build", "dash_workspace_size", "load", "params", "route_out", "DecodeState",
           "Prefill", "prefill", "dash_decode_paged", "dash_summary_append_paged", "dash_summary_build_paged",
           "paged_kv", "PagedDecodeState"]
