"""B200-native multi-scale deformable attention core (MSDeformAttn), forward and
training backward, as hand-written sm_100a CUDA kernels behind a C ABI.

``forward`` / ``backward`` / ``ms_deform_attn`` (and the ``fused_*`` variants fed
with raw reference points, offsets and logits) marshal torch tensors into the
C-ABI library ``libmsda.so`` (built in-tree by ``csrc/build.py``).  Every
step of the operator runs in the CUDA kernels; there is no CPU or PyTorch
fallback.  Importing this package loads neither torch nor the library: the
binding is imported on first attribute access, and the library on the first
call, which raises if it is missing.
"""
_BINDING_NAMES = ("forward", "backward", "ms_deform_attn", "MSDeformAttnFunction",
                  "fused_forward", "fused_backward", "ms_deform_attn_fused",
                  "MSDeformAttnFusedFunction", "output_projection", "MSDAError", "library")

__all__ = list(_BINDING_NAMES)


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
