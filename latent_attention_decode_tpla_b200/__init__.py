"""TPLA decode (Tensor-Parallel Latent Attention) for NVIDIA B200 (sm_100a).

The compute lives in ``libtpla.so`` (hand-written CUDA, C ABI declared in
``include/tpla.h``).  ``latent_attention_decode_tpla_b200.tpla`` is the thin
ctypes binding; the library is loaded on first use and a missing library is
an error, never a fallback.
"""

__all__ = ["tpla", "inputs"]
