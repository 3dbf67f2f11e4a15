"""The C ABI library loads on a machine without a GPU, exports every function
that include/bfmoe.h declares, and rejects bad arguments on the host before
touching the device."""
import ctypes

import pytest

from ternary_butterfly_experts_b200 import build, capi


@pytest.fixture(scope="module")
def L():
    build.build()
    return capi.lib()


def test_exports_every_declared_symbol(L):
    names = capi.header_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(L, n), f"{n} declared in bfmoe.h but not exported"
        assert n in capi.SIGNATURES, f"{n} has no ctypes signature"


def test_workspace_size_host_only(L):
    a = L.bfmoe_workspace_size(512, 256, 16384, 2, capi.BFMOE_BF16)
    b = L.bfmoe_workspace_size(512, 256, 16384, 2, capi.BFMOE_F32)
    assert a > 0 and b > a and a % 256 == 0
    assert L.bfmoe_workspace_size(500, 256, 16384, 2, 1) == 0      # not a power of two
    assert L.bfmoe_workspace_size(512, 4, 10, 5, 1) == 0           # k > N
    assert L.bfmoe_workspace_size(512, 4, 10, 9, 1) == 0           # k > 8
    assert L.bfmoe_workspace_size(512, 4, 10, 2, 7) == 0           # bad dtype
    assert L.bfmoe_workspace_size(8192, 4, 10, 2, 1) == 0          # d too large


def test_argument_checks_before_any_launch(L):
    n0 = L.bfmoe_launch_count()
    assert L.bfmoe_pack_base(None, 64, None, None) == capi.BFMOE_EINVAL
    assert b"NULL" in L.bfmoe_last_error()
    assert L.bfmoe_pack_base(ctypes.c_void_p(16), 48, ctypes.c_void_p(16), None) == capi.BFMOE_EINVAL
    lay = capi.BfmoeLayer(64, 4, 16, ctypes.c_float(0.1), 16, 16)
    assert L.bfmoe_forward(ctypes.byref(lay), None, 1, 4, 2, None, None, None, None, None, None, 0,
                           None) == capi.BFMOE_EINVAL
    assert L.bfmoe_forward(ctypes.byref(lay), 16, 1, 4, 5, 16, 16, 16, 16, 16, None, 0, None) == capi.BFMOE_EINVAL
    assert L.bfmoe_forward(None, 16, 1, 4, 2, 16, 16, 16, 16, 16, None, 0, None) == capi.BFMOE_EINVAL
    # a workspace that is missing or too small is reported as such
    assert L.bfmoe_forward(ctypes.byref(lay), 16, 1, 4, 2, 16, 16, 16, 16, 16, None, 0,
                           None) == capi.BFMOE_EWORKSPACE
    assert L.bfmoe_forward(ctypes.byref(lay), 16, 1, 4, 2, 16, 16, 16, 16, 16, 256, 10,
                           None) == capi.BFMOE_EWORKSPACE
    assert L.bfmoe_forward(ctypes.byref(lay), 16, 1, 4, 2, 16, 16, 16, 16, 16, 258, 1 << 30,
                           None) == capi.BFMOE_EWORKSPACE   # misaligned
    assert L.bfmoe_router_topk(16, 1, 4, 64, 16, None, 4, 0, 16, 16, 16, 16, 16, None, 0,
                               None) == capi.BFMOE_EINVAL     # k = 0
    assert L.bfmoe_materialize_expert(ctypes.byref(lay), 4, 16, None) == capi.BFMOE_EINVAL
    assert L.bfmoe_unpack_base(16, 100, 16, None) == capi.BFMOE_EINVAL
    assert L.bfmoe_launch_count() == n0


def test_binding_names_match_header():
    import ternary_butterfly_experts_b200 as B
    for n in capi.header_functions():
        assert hasattr(B, n), f"binding lacks {n}"


def test_host_call_checks_before_any_launch(L):
    n0 = L.bfmoe_launch_count()
    lay = capi.BfmoeLayer(64, 4, 16, ctypes.c_float(0.1), 16, 16)
    f = L.bfmoe_moe_forward_host
    assert f(None, 16, 1, 300, 16, None, 2, 16, 0, 256, 1 << 30, None) == capi.BFMOE_EINVAL       # no layer
    assert f(ctypes.byref(lay), 16, 1, 300, 16, None, 5, 16, 0, 256, 1 << 30, None) == capi.BFMOE_EINVAL  # k > N
    assert f(ctypes.byref(lay), None, 1, 300, 16, None, 2, 16, 0, 256, 1 << 30, None) == capi.BFMOE_EINVAL
    assert f(ctypes.byref(lay), 16, 1, 300, 16, None, 2, None, 0, 256, 1 << 30, None) == capi.BFMOE_EINVAL
    assert f(ctypes.byref(lay), 16, 3, 300, 16, None, 2, 16, 0, 256, 1 << 30, None) == capi.BFMOE_EINVAL  # dtype
    assert f(ctypes.byref(lay), 16, 1, 300, 16, None, 2, 16, 0, None, 0, None) == capi.BFMOE_EWORKSPACE
    assert f(ctypes.byref(lay), 16, 1, 300, 16, None, 2, 16, 0, 256, 100, None) == capi.BFMOE_EWORKSPACE
    assert f(ctypes.byref(lay), 16, 1, 300, 16, None, 2, 16, 0, 264, 1 << 30, None) == capi.BFMOE_EWORKSPACE
    assert f(ctypes.byref(lay), 16, 1, 0, 16, None, 2, 16, 0, None, 0, None) == capi.BFMOE_OK  # T = 0: nothing to do
    assert L.bfmoe_launch_count() == n0


def test_host_workspace_size(L):
    bf = capi.BFMOE_BF16
    full = L.bfmoe_moe_host_workspace_size(512, 256, 16384, 2, bf, 0)
    one = L.bfmoe_moe_workspace_size(512, 256, 2816, 2, bf)
    # device x and y for all tokens plus, per compute stream, one default
    # chunk's scratch (four chunks of 4096 tokens here, two streams)
    assert full >= 2 * 16384 * 512 * 2 + 2 * L.bfmoe_moe_workspace_size(512, 256, 4096, 2, bf) and full % 256 == 0
    assert full >= 2 * 16384 * 512 * 2 + one
    # one chunk of all tokens: one compute stream with the whole call's scratch
    big = L.bfmoe_moe_host_workspace_size(512, 256, 16384, 2, bf, 16384)
    assert big >= 2 * 16384 * 512 * 2 + L.bfmoe_moe_workspace_size(512, 256, 16384, 2, bf)
    assert L.bfmoe_moe_host_workspace_size(500, 256, 16384, 2, bf, 0) == 0
    assert L.bfmoe_moe_host_workspace_size(512, 4, 100, 5, bf, 0) == 0


def test_router_rejects_partial_bucket_outputs():
    """counts, offsets and rows: all given or all NULL (checked before any launch)."""
    import ctypes
    L = capi.lib()
    buf = ctypes.create_string_buffer(64)
    p = ctypes.cast(buf, ctypes.c_void_p)
    rc = L.bfmoe_router_topk(p, 1, 0, 64, p, None, 4, 2, p, p, p, None, None, p, 64, None)
    assert rc == 1  # BFMOE_EINVAL
    assert b"all given or all NULL" in L.bfmoe_last_error()


def test_prepare_gate_sizes_and_argument_checks():
    """bfmoe_gate_parts_size and bfmoe_prepare_gate's checks (before any launch)."""
    import ctypes
    L = capi.lib()
    assert L.bfmoe_gate_parts_size(256, 512) == 3 * 256 * 512 * 2
    assert L.bfmoe_gate_parts_size(0, 512) == 0 and L.bfmoe_gate_parts_size(4, 100) == 0
    assert L.bfmoe_prepare_gate(None, 4, 64, 256, 1 << 20, None) == capi.BFMOE_EINVAL
    assert L.bfmoe_prepare_gate(16, 4, 63, 256, 1 << 20, None) == capi.BFMOE_EINVAL
    assert L.bfmoe_prepare_gate(16, 4, 64, 16, 1 << 20, None) == capi.BFMOE_EWORKSPACE   # not 256-byte aligned
    assert L.bfmoe_prepare_gate(16, 4, 64, 256, 100, None) == capi.BFMOE_EWORKSPACE      # too small


def test_decode_forward_argument_checks():
    import ctypes
    L = capi.lib()
    lay = capi.BfmoeLayer(64, 4, 16, ctypes.c_float(0.1), 16, 16)
    f = L.bfmoe_decode_forward
    assert f(None, 16, 1, 4, 2, 16, 16, 16, None) == capi.BFMOE_EINVAL                 # no layer
    assert f(ctypes.byref(lay), 16, 1, 4, 5, 16, 16, 16, None) == capi.BFMOE_EINVAL    # k > N
    assert f(ctypes.byref(lay), 16, 7, 4, 2, 16, 16, 16, None) == capi.BFMOE_EINVAL    # bad dtype
    assert f(ctypes.byref(lay), None, 1, 4, 2, 16, 16, 16, None) == capi.BFMOE_EINVAL  # NULL x
    assert f(ctypes.byref(lay), None, 1, 0, 2, None, None, None, None) == capi.BFMOE_OK  # T = 0: nothing to do
