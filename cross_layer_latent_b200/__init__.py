"""LatentIndex decode indexer on B200 (sm_100a).

The compute lives in libli.so (C ABI in include/li.h); this package is the
thin Python binding over it (``_binding``) plus ``GroupIndexer``, which wires
the entry points into one layer group's decode step.  Importing fails when the
library has not been built: there is no CPU fallback.
"""
from ._binding import (EXPORTED, LI_BF16, LI_E4M3, LI_F32, STATUS_NAMES, Cache, Context, LatentTransform, LiError,
                       Query, li_absorb_query, li_absorb_query_group, li_append_latent, li_append_latent_ex,
                       li_attention_recall, li_create, li_destroy, li_device_status, li_dsa_score_topk, li_hs_anchor_candidates, li_hs_follower_refine,
                       li_profile_enable, li_profile_read, li_profile_reset, li_score_topk, li_score_topk_static,
                       li_set_trace, li_set_wait_limit, li_status_string, li_topk, li_workspace_bytes, workspace)
from .group import GroupIndexer

__all__ = ["Cache", "Context", "LatentTransform", "LiError", "Query", "LI_BF16", "LI_E4M3", "LI_F32",
           "STATUS_NAMES", "EXPORTED", "li_absorb_query", "li_absorb_query_group", "li_append_latent",
           "li_append_latent_ex", "li_attention_recall", "li_create", "li_destroy", "li_device_status", "li_dsa_score_topk", "li_hs_anchor_candidates",
           "li_hs_follower_refine", "li_profile_enable", "li_profile_read", "li_profile_reset", "li_score_topk",
           "li_score_topk_static", "li_set_trace", "li_set_wait_limit", "li_status_string", "li_topk",
           "li_workspace_bytes", "workspace", "GroupIndexer"]
