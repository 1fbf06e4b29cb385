"""MXFP4 attention for NVIDIA B200 (sm_100a): a C-ABI CUDA library (libmxattn.so) with a thin
torch binding. Importing the package does not load the CUDA library; the first call does, and
fails loudly if it has not been built."""
from .api import (SCALE_OCP, SCALE_UOS, OUT_F32, OUT_BF16, mxattn_quantize, mxattn_forward,  # noqa: F401
                  mxattn_forward_prepare, mxattn_forward_attend, mxattn_forward_debug,
                  mxattn_check_status, workspace_size, alloc_workspace, npad)

__all__ = ["SCALE_OCP", "SCALE_UOS", "OUT_F32", "OUT_BF16", "mxattn_quantize", "mxattn_forward",
           "mxattn_forward_prepare", "mxattn_forward_attend", "mxattn_forward_debug",
           "mxattn_check_status", "workspace_size", "alloc_workspace", "npad"]
