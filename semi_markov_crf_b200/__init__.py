"""B200-native streaming semi-CRF forward-backward (Flash-SemiCRF method).

The compute path is the C-ABI library ``libsemicrf_b200.so`` (hand-written
sm_100a CUDA kernels, declared in ``include/semicrf.h``); ``semicrf`` is its
thin Python binding.  ``synth`` draws the seeded synthetic workloads.

Importing the package does not load the CUDA library; touching any binding
name does, and fails loudly if the library has not been built.
"""

from __future__ import annotations

_BINDING_NAMES = {
    "workspace_bytes", "prefix_center", "forward", "backward", "viterbi", "get_status",
    "strerror", "SemiCRFError", "library_path", "Workspace", "FLAG_NO_CENTER",
    "FLAG_FORWARD_ONLY", "selftest_bounded_wait", "forward_noalloc", "profile_enable",
    "profile_read",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import semicrf
        return getattr(semicrf, name)
    raise AttributeError(name)
