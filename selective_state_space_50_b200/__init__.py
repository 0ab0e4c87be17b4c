"""B200-native selective scan (S6): a C-ABI CUDA library for sm_100a
(libssmscan.so, declared in include/ssm_scan.h) and a thin Python binding.

    from selective_state_space_50_b200 import selective_scan_fwd, selective_scan_bwd
"""
from .ssm_scan import (SSMError, load_library, selective_scan_bwd,  # noqa: F401
                       selective_scan_fwd)

__all__ = ["selective_scan_fwd", "selective_scan_bwd", "load_library", "SSMError"]
