"""Frame-wise Gated DeltaNet frame scan for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libgdn.so`` (``include/gdn.h``); ``api`` is a thin
PyTorch binding (argument marshalling only). Accessing any API name loads the library and
raises ImportError if it has not been built (``python -m frame_wise_gated_deltanet_b200.build``);
there is no CPU fallback.
"""
_API = (
    "gdn_frame_forward",
    "gdn_frame_forward_rope",
    "gdn_frame_step",
    "gdn_frame_backward",
    "gdn_frame_forward_train",
    "gdn_frame_backward_saved",
    "gdn_train_saved_bytes",
    "gdn_rope_3d",
    "gdn_softmax_attention",
    "gdn_frame_stats",
    "gdn_block_causal_la",
    "gdn_sync_status",
    "gdn_release_workspace",
    "gdn_workspace_bytes",
    "gdn_la_workspace_bytes",
    "gdn_backward_workspace_bytes",
    "GdnError",
)
__all__ = list(_API)


def __getattr__(name):
    if name in _API:
        from . import api
        return getattr(api, name)
    raise AttributeError(name)
