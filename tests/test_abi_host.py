"""Host-side tests of the C ABI: the library loads, exports what include/gdn.h
declares, sizes workspaces, and rejects bad arguments before launching
anything (these calls never touch a GPU: validation fails first)."""
import ctypes
import os
import re

import pytest

import gated_delta_rule_99_b200 as gdn
from gated_delta_rule_99_b200 import _binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x7F0000000000  # a 256-byte aligned address that is never dereferenced


def header_functions():
    src = open(os.path.join(ROOT, "include", "gdn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol():
    L = gdn.lib()
    names = header_functions()
    assert set(names) == set(B.EXPORTS)
    for n in names:
        assert hasattr(L, n), n


def test_version_and_chunk():
    assert gdn.lib().gdn_version() >= 100
    assert gdn.lib().gdn_chunk_size() == 64


def test_status_strings():
    L = gdn.lib()
    for code, s in B.STATUS.items():
        assert L.gdn_status_string(code).decode() == s
    assert L.gdn_status_string(99).decode() == "unknown status"


@pytest.mark.parametrize("bad,code", [
    (dict(dk=96), 2), (dict(dv=32), 2), (dict(dk=512), 2), (dict(dv=192), 2), (dict(dtype=7), 2),
    (dict(B=0), 1), (dict(H=0), 1),
    (dict(T=-1), 1), (dict(n_seqs=3, B=2), 1), (dict(B=1 << 20, T=1 << 12), 1)])
def test_workspace_size_rejects_bad_descriptors(bad, code):
    args = dict(B=2, T=100, H=3, dk=64, dv=128, n_seqs=0, dtype=0, scale=1.0)
    args.update(bad)
    d = gdn.make_desc(**args)
    assert gdn.fwd_workspace_size(d) == 0 and gdn.bwd_workspace_size(d) == 0
    rc = _fwd(d, ws_bytes=1 << 40)
    assert rc == code


def test_head_dim_256_takes_the_cuda_core_layout_for_both_dtypes():
    """d = 256 runs on the fp32 CUDA-core kernels whatever the dtype: its workspace
    is that path's (fp32 intermediates and scratch slots with 256-float rows), the
    same for bf16 and fp32 inputs, and larger than at d = 128."""
    for K, V in ((256, 256), (256, 128), (64, 256)):
        w = [gdn.fwd_workspace_size(gdn.make_desc(2, 100, 3, K, V, dtype=dt)) for dt in (0, 1)]
        b = [gdn.bwd_workspace_size(gdn.make_desc(2, 100, 3, K, V, dtype=dt)) for dt in (0, 1)]
        assert w[0] == w[1] > 0 and b[0] == b[1] > w[0]
    small = gdn.fwd_workspace_size(gdn.make_desc(2, 100, 3, 128, 128, dtype=1))
    assert gdn.fwd_workspace_size(gdn.make_desc(2, 100, 3, 256, 256, dtype=1)) > small


def test_flags_match_header_and_unknown_bits_are_rejected():
    import re
    hdr = open(os.path.join(ROOT, "include", "gdn.h")).read()
    defs = dict(re.findall(r"#define (GDN_FLAG_\w+) (\d+)", hdr))
    assert int(defs["GDN_FLAG_PIECE_SCAN"]) == gdn.GDN_FLAG_PIECE_SCAN
    assert int(defs["GDN_FLAG_QK_L2NORM"]) == gdn.GDN_FLAG_QK_L2NORM
    assert int(defs["GDN_FLAG_VALUE_SLICES"]) == gdn.GDN_FLAG_VALUE_SLICES
    every = gdn.GDN_FLAG_QK_L2NORM | gdn.GDN_FLAG_PIECE_SCAN | gdn.GDN_FLAG_VALUE_SLICES
    ok = gdn.make_desc(2, 100, 3, 64, 128, flags=every)
    assert gdn.fwd_workspace_size(ok) > 0
    bad = gdn.make_desc(2, 100, 3, 64, 128, flags=8)
    assert gdn.fwd_workspace_size(bad) == 0 and _fwd(bad, ws_bytes=1 << 40) == 1


def test_l2norm_workspace_holds_normalised_copies_only_off_the_tensor_core_path():
    for dt, K, V, grows in ((1, 64, 128, True), (1, 128, 128, True), (0, 64, 64, False),
                            (0, 128, 128, False)):
        plain = gdn.make_desc(2, 300, 3, K, V, dtype=dt)
        l2 = gdn.make_desc(2, 300, 3, K, V, dtype=dt, flags=gdn.GDN_FLAG_QK_L2NORM)
        for size in (gdn.fwd_workspace_size, gdn.bwd_workspace_size):
            a, b = size(plain), size(l2)
            if grows:  # two copies of (B*T*H, K) rows in the input dtype plus two norm vectors
                es = 4 if dt == 1 else 2
                assert b - a >= 2 * 2 * 300 * 3 * K * es + 2 * 4 * 2 * 300 * 3
            else:
                assert a == b


def test_workspace_sizes_grow():
    a = gdn.fwd_workspace_size(gdn.make_desc(1, 64, 1, 64, 64))
    b = gdn.fwd_workspace_size(gdn.make_desc(1, 128, 1, 64, 64))
    c = gdn.bwd_workspace_size(gdn.make_desc(1, 128, 1, 64, 64))
    assert 0 < a < b <= c
    for dt in (0, 1):
        d = gdn.make_desc(4, 4096, 16, 128, 128, dtype=dt)
        assert gdn.bwd_workspace_size(d) >= gdn.fwd_workspace_size(d) > 0


def _fwd(d, ws_bytes=None, ptrs=None, cu=None, cu_host=None, ws=FAKE):
    L = gdn.lib()
    p = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, h0=None, o=FAKE, hT=None)
    p.update(ptrs or {})
    if ws_bytes is None:
        ws_bytes = gdn.fwd_workspace_size(d)
    return L.gdn_fwd(ctypes.byref(d), p["q"], p["k"], p["v"], p["g"], p["beta"], cu, cu_host,
                     p["h0"], p["o"], p["hT"], ws, ws_bytes, None)


def _bwd(d, ptrs=None, ws_bytes=None):
    L = gdn.lib()
    names = ("q", "k", "v", "g", "beta", "h0", "do", "dhT", "dq", "dk", "dv", "dg", "dbeta", "dh0")
    p = {n: FAKE for n in names}
    p.update(h0=None, dhT=None, dh0=None)
    p.update(ptrs or {})
    if ws_bytes is None:
        ws_bytes = gdn.bwd_workspace_size(d)
    return L.gdn_bwd(ctypes.byref(d), p["q"], p["k"], p["v"], p["g"], p["beta"], None, None,
                     p["h0"], p["do"], p["dhT"], p["dq"], p["dk"], p["dv"], p["dg"], p["dbeta"],
                     p["dh0"], FAKE, ws_bytes, None)


def test_null_and_misaligned_pointers():
    d = gdn.make_desc(2, 100, 3, 64, 128)
    assert _fwd(d, ptrs=dict(q=None)) == 1
    assert _fwd(d, ptrs=dict(o=None)) == 1
    assert _fwd(d, ptrs=dict(v=FAKE + 8)) == 3
    assert _fwd(d, ptrs=dict(hT=FAKE + 4)) == 3
    assert _fwd(d, ws=FAKE + 16) == 3
    assert _fwd(d, ws=None) == 4
    assert _bwd(d, ptrs=dict(dbeta=None)) == 1
    assert _bwd(d, ptrs=dict(do=None)) == 1
    assert _bwd(d, ptrs=dict(dh0=FAKE + 2)) == 3


def test_workspace_too_small():
    d = gdn.make_desc(2, 100, 3, 64, 128)
    assert _fwd(d, ws_bytes=gdn.fwd_workspace_size(d) - 1) == 4
    assert _bwd(d, ws_bytes=gdn.bwd_workspace_size(d) - 1) == 4


def _cu(vals):
    arr = (ctypes.c_int32 * len(vals))(*vals)
    return arr


@pytest.mark.parametrize("cu", [[0, 50, 40, 100], [1, 50, 100], [0, 50, 99], [0, 50, 101]])
def test_bad_seqlens_rejected_on_host(cu):
    d = gdn.make_desc(1, 100, 2, 64, 64, n_seqs=len(cu) - 1)
    host = _cu(cu)
    assert _fwd(d, cu=FAKE, cu_host=ctypes.cast(host, ctypes.c_void_p)) == 1


def test_seqlens_require_single_row_and_device_copy():
    d = gdn.make_desc(1, 100, 2, 64, 64, n_seqs=2)
    host = _cu([0, 40, 100])
    assert _fwd(d, cu=None, cu_host=ctypes.cast(host, ctypes.c_void_p)) == 1
    dense = gdn.make_desc(1, 100, 2, 64, 64)
    assert _fwd(dense, cu=FAKE, cu_host=ctypes.cast(host, ctypes.c_void_p)) == 1


def test_python_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(1, 8, 1, 64, dtype=torch.bfloat16)
    g = torch.zeros(1, 8, 1)
    with pytest.raises(ValueError):
        gdn.gdn_fwd(x, x, x, g, g)


def test_decode_rejects_bad_arguments():
    L = gdn.lib()
    p = [FAKE] * 5
    ok = gdn.make_desc(4, 1, 2, 128, 128)
    st = FAKE
    assert L.gdn_decode(ctypes.byref(gdn.make_desc(4, 1, 2, 96, 128)), *p, st, FAKE, None) == 2
    assert L.gdn_decode(ctypes.byref(gdn.make_desc(4, 1, 2, 256, 128)), *p, st, FAKE, None) == 2
    assert L.gdn_decode(ctypes.byref(gdn.make_desc(4, 0, 2, 128, 128)), *p, st, FAKE, None) == 1
    assert L.gdn_decode(ctypes.byref(gdn.make_desc(1, 1, 2, 128, 128, n_seqs=1)), *p, st, FAKE,
                        None) == 1
    assert L.gdn_decode(ctypes.byref(ok), *p, None, FAKE, None) == 1
    assert L.gdn_decode(ctypes.byref(ok), *p, FAKE + 4, FAKE, None) == 3


def test_testing_hooks_match_header_and_are_callable_without_a_gpu():
    hdr = open(os.path.join(ROOT, "include", "gdn.h")).read()
    defs = dict(re.findall(r"#define (GDN_TEST_\w+) (\d+)", hdr))
    assert int(defs["GDN_TEST_STALL_COPY"]) == gdn.GDN_TEST_STALL_COPY
    assert int(defs["GDN_TEST_FAIL_LAUNCH"]) == gdn.GDN_TEST_FAIL_LAUNCH
    # per-thread settings only: setting and clearing them touches no device
    gdn.set_wait_limit(1000)
    gdn.set_test_hook(gdn.GDN_TEST_FAIL_LAUNCH)
    gdn.set_test_hook(0)
    gdn.set_wait_limit(0)
    # an argument error still comes first, hook or not
    gdn.set_test_hook(gdn.GDN_TEST_FAIL_LAUNCH)
    try:
        assert _fwd(gdn.make_desc(B=0, T=10, H=1, dk=64, dv=64), ws_bytes=1 << 20) == 1
    finally:
        gdn.set_test_hook(0)


def test_descriptor_products_are_range_checked_before_they_are_formed():
    # B * T would overflow a signed 64-bit product; both are rejected first
    for B, T in ((1 << 40, 1 << 40), (3, (1 << 62)), (1 << 62, 2)):
        d = gdn.make_desc(B=B, T=T, H=1, dk=64, dv=64)
        assert gdn.fwd_workspace_size(d) == 0
    # (chunk, head) grids must stay within int32
    d = gdn.make_desc(B=1, T=(1 << 31) - 64, H=1 << 10, dk=64, dv=64)
    assert gdn.fwd_workspace_size(d) == 0
