"""Exact scaled dot-product attention (forward + backward) for B200 / sm_100a.

The computation runs in libfa.so (hand-written tcgen05/TMEM/TMA kernels behind
the C ABI declared in include/fa.h); ``api`` is the thin Python binding.
"""
import importlib

__version__ = "0.1.0"

_API_NAMES = ("fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_last_device_status", "fa_set_softmax_options",
              "fa_exp2_eval", "fa_strerror", "fa_version", "fa_profile_next", "fa_bwd_noalloc", "fa_set_forward_variant",
              "fa_set_backward_variant", "fa_sm_clock_probe",
              "fa_fwd_qk", "fa_bwd_qk", "fa_bwd_qk_workspace_size", "fa_lse_merge", "fa_accumulate_bf16",
              "fa_convert_f32_bf16")


def __getattr__(name):
    # the binding imports torch; load it lazily so the input generator can be
    # imported on its own
    if name in _API_NAMES:
        return getattr(importlib.import_module(__name__ + ".api"), name)
    raise AttributeError(name)
