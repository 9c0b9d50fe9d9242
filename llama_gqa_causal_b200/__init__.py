"""B200-native LLaMA self-attention: RoPE + GQA/MQA/MHA prefill and KV-cache decode.

The compute path lives in the C-ABI library ``libllama_attn.so`` (hand-written
sm_100a CUDA kernels); ``api`` is a thin ctypes binding with the same entry
point names.  Importing this package does not load the library; the first call
into ``api`` does, and raises if it is missing.
"""
__all__ = ["api", "workloads"]
