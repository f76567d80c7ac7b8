"""SageAttention-style low-bit attention forward for B200 (sm_100a).

Per head: K is smoothed by its per-channel token mean; Q is quantised to INT8 per
128-token block and K per 64-token block (scale = max|x|/127, round-half-even);
S = q_i8 . k_i8^T runs exactly in int32 on tcgen05 tensor cores with the accumulator in
tensor memory; the online softmax runs in fp32; P is scaled by 448 and cast to FP8 e4m3;
V is cast to FP8 e4m3 per channel; P.V accumulates in fp32.  An optional keep-mask over
128-query x 64-key blocks skips masked blocks without loading them.

The compute lives in the C-ABI library ``libsa.so`` (``include/sa.h``); the functions
re-exported here (``sa_quantize_qk``, ``sa_quantize_v``, ``sa_attn_fwd`` ...) only marshal
torch tensors into it.  Importing them raises if the library has not been built: there
is no CPU fallback.
"""

_BINDING_NAMES = (
    "sa_quantize_qk", "sa_quantize_v", "sa_attn_fwd", "sa_attn_fwd_quantized",
    "sa_debug_qk_s32", "sa_get_device_status", "sa_status_string", "sa_workspace_bytes",
    "sa_release_workspace", "SAError", "library_path",
)


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
