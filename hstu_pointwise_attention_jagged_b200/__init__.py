"""B200 (sm_100a) forward pass of jagged, target-aware HSTU pointwise (SiLU) attention.

    out = Mask(SiLU(alpha * Q K^T)) V / N

over jagged batches of user-interaction histories with appended candidate tokens (history
causal, each candidate sees all history plus itself), plus the streaming variant that queries
only new tokens against a cached K/V prefix.  The work happens in ``libhstu_attn.so`` (C ABI in
``include/hstu_attn.h``); :mod:`.binding` marshals torch tensors into it.  The binding's names
are re-exported lazily so that :mod:`.workloads` and :mod:`.metrics` import without it.
"""
_BINDING_NAMES = ("HstuError", "hstu_attn_fwd", "hstu_attn_fwd_cached", "hstu_attn_fwd_rab", "hstu_attn_plan_bytes", "hstu_attn_plan",
                  "hstu_attn_fwd_planned", "hstu_attn_fwd_noalloc", "hstu_attn_get_error", "hstu_attn_status_string",
                  "hstu_attn_selfcheck_wait_timeout", "hstu_attn_gemm_bf16", "hstu_attn_bwd", "hstu_attn_bwd_workspace_limit", "hstu_attn_partition", "shard_of", "hstu_layer_workspace_bytes",
                  "hstu_layer_fwd", "hstu_layers_fwd", "plan_contents",
                  "library_path", "load_library")


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
