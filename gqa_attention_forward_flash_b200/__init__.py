"""B200-native (sm_100a) grouped-query-attention forward.

The computation lives in ``libgqa_attn.so`` (hand-written CUDA, C ABI in
``include/gqa_attn.h``); :mod:`.binding` marshals torch tensors to it.
"""
from .binding import (GQAError, gqa_attention_fwd, gqa_attention_fwd_partial, gqa_get_device_error,  # noqa: F401
                      gqa_splitkv_combine, gqa_status_string, gqa_version, load)
