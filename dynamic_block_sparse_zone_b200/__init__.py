"""B200 (sm_100a) implementation of Prism's dynamic sparse video self-attention.

The computation lives in libprism.so (CUDA, C ABI in include/prism.h);
``binding`` marshals torch tensors into it.  ``synth`` draws seeded inputs.
"""
from .binding import (PrismError, PrismPlan, Params, gather_sequence, heads_to_sequence, load_library, params_for,
                      prism_attn_bwd, sequence_to_heads,
                      prism_attn_fwd, prism_attn_fwd_taylor, prism_plan_build, prism_plan_bytes, prism_plan_create,
                      prism_plan_destroy)

__all__ = ["PrismError", "PrismPlan", "Params", "gather_sequence", "heads_to_sequence", "load_library", "params_for",
           "prism_attn_bwd", "sequence_to_heads",
           "prism_attn_fwd", "prism_attn_fwd_taylor", "prism_plan_build", "prism_plan_bytes", "prism_plan_create",
           "prism_plan_destroy"]
