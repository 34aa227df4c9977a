"""B200-native gated delta rule (Gated DeltaNet token mixer).

The compute path is ``libgdn.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in ``include/gdn.h``); ``binding`` marshals torch tensors into it.  The
binding is imported on first use of one of its names, so that
``gated_delta_rule_130_b200.inputs`` can be used without the CUDA library; the
first such use raises if ``libgdn.so`` is missing -- there is no fallback.
"""

_BINDING_NAMES = {
    "chunk_fwd", "chunk_fwd_varlen", "chunk_fwd_varlen_workspace_size", "decode_step",
    "chunk_fwd_workspace_size", "chunk_fwd_path", "library_path", "chunk_bwd",
    "chunk_bwd_workspace_size", "chunk_fwd_cw", "chunk_fwd_cw_workspace_size", "decode_step_cw",
    "GdnError", "check_device_status",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
