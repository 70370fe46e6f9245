"""libcausalattn: multi-head causal self-attention forward/backward for B200 (sm_100a).

The compute path is the C-ABI shared library libcausalattn.so (hand-written
tcgen05/TMA kernels); `abi` is its ctypes binding, `inputs` the seeded
synthetic input recipe.
"""
from . import abi  # noqa: F401
from .abi import (attention_backward, attention_forward, causal_attention,  # noqa: F401
                  gpt_attn_bwd, gpt_attn_bwd_dkdv, gpt_attn_bwd_dq, gpt_attn_bwd_preprocess,
                  gpt_attn_fwd)
