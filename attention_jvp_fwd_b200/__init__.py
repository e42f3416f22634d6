"""B200-native attention forward + JVP (the rCM / sCM hot path).

``attn_jvp_fwd`` returns O = softmax(s Q K^T) V, its tangent O' along
(Q', K', V') and the row log-sum-exp, computed by hand-written sm_100a
kernels behind a small C ABI (``include/attn_jvp.h``).  Importing this package
does not load the CUDA library; the first call does, and fails loudly if it
has not been built.  ``scm_tangent_loss`` is the tangent-normalised sCM loss
term that consumes such tangents, and ``qkv_rmsnorm_jvp`` the projection + RMSNorm
layer that produces attention's inputs and their tangents.
"""
from .api import (ATTN_JVP_ERR_ALIGN, ATTN_JVP_ERR_HEADDIM, ATTN_JVP_ERR_LAUNCH,  # noqa: F401
                  ATTN_JVP_ERR_NULL, ATTN_JVP_ERR_SHAPE, ATTN_JVP_ERR_TIMEOUT,
                  ATTN_JVP_ERR_VALUE, ATTN_JVP_OK, AttnJvpError, attn_jvp_check,
                  attn_jvp_fwd, attn_jvp_fwd_trace, attn_jvp_status_string, attn_jvp_workspace_bytes,
                  library_path,
                  qkv_prologue_check, qkv_rmsnorm_jvp, scm_tangent_loss)

__all__ = ["attn_jvp_fwd", "attn_jvp_fwd_trace", "attn_jvp_workspace_bytes", "attn_jvp_check", "attn_jvp_status_string",
           "AttnJvpError", "library_path", "scm_tangent_loss", "qkv_rmsnorm_jvp", "qkv_prologue_check"]
