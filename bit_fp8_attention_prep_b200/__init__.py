"""VC-Attention forward hot path for one B200 (sm_100a).

The compute path is the C-ABI library ``libvcattn.so`` built from ``csrc/``;
``vc_attn`` (the binding) marshals torch tensors into its calls. Importing this
package does not load the library; the first call into ``vc_attn`` does, and
fails loudly if it is missing.
"""
__all__ = ["vc_attn", "synth"]
