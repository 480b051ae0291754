"""B200-native (sm_100a) chunkwise Gated DeltaNet layer, forward and backward.

The compute lives in libgdn.so (CUDA kernels behind the C ABI in
include/gdn.h); this package is its thin Python binding plus the seeded
synthetic-input generator.  Importing it does not load the library; the first
call does, and raises if the library was not built.
"""
from ._binding import (EXPORTS, GDN_BF16, GDN_FLAG_PIECE_SCAN, GDN_FLAG_QK_L2NORM,  # noqa
                       GDN_FLAG_VALUE_SLICES, GDN_FP32,
                       GDN_TEST_FAIL_LAUNCH, GDN_TEST_STALL_COPY, GdnDesc, GdnError, LaunchTrace,
                       alloc_workspace, bwd_workspace_size, device_status, fwd_workspace_size,
                       gdn_bwd, gdn_decode, gdn_fwd, lib, make_desc, set_test_hook,
                       set_wait_limit)

__all__ = ["gdn_fwd", "gdn_bwd", "gdn_decode", "device_status", "fwd_workspace_size",
           "bwd_workspace_size", "alloc_workspace", "LaunchTrace", "make_desc", "GdnDesc",
           "GdnError", "lib", "GDN_BF16", "GDN_FP32", "GDN_FLAG_PIECE_SCAN", "GDN_FLAG_QK_L2NORM",
           "GDN_FLAG_VALUE_SLICES",
           "GDN_TEST_STALL_COPY", "GDN_TEST_FAIL_LAUNCH", "set_wait_limit", "set_test_hook",
           "EXPORTS"]
