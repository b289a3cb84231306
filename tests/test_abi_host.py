"""C-ABI checks that need no GPU: the library builds/loads, exports every symbol the header
declares, and rejects invalid arguments on the host before anything is enqueued."""
import ctypes
import os
import re

import pytest

import quantized_expert_ffn_gemm_b200 as moe
from quantized_expert_ffn_gemm_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_ffn.h")

FAKE = ctypes.c_void_p(0x10000)      # aligned, never dereferenced: every call below fails validation first
FAKE_MIS = ctypes.c_void_p(0x10008)  # 8-byte aligned only


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(moe_[a-z_0-9]+)\s*\(", text, re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["moe_router_topk", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_layer_forward",
              "moe_stack_forward", "moe_dequant_rows", "moe_read_device_error", "moe_workspace_bytes"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n
    assert sorted(declared_functions()) == sorted(moe.EXPORTED)


def test_status_strings(lib):
    assert moe.status_string(0) == "MOE_OK"
    assert moe.status_string(7) == "MOE_ERR_TIMEOUT"
    assert moe.status_string(99) == "MOE_ERR_UNKNOWN"


def test_workspace_bytes(lib):
    assert moe.workspace_bytes(2048, 512, 10, 512, True, 8192) > 8192 * 11 * 2048 * 2 * 2
    assert moe.workspace_bytes(2048, 512, 10, 512, True, 1) > 0
    assert moe.workspace_bytes(2040, 512, 10, 512, True, 1) == 0   # H not a multiple of 64
    assert moe.workspace_bytes(2048, 512, 0, 512, True, 1) == 0    # k = 0
    assert moe.workspace_bytes(2048, 8, 9, 512, True, 1) == 0      # k > E
    assert moe.workspace_bytes(2048, 512, 33, 512, True, 1) == 0   # k > 32
    assert moe.workspace_bytes(2048, 512, 10, 512, True, -1) == 0


def _desc(H=2048, E=512, k=10, I=512, sh=0):
    return moe.LayerDesc(H, E, k, I, sh)


def _set(H=2048, E=512, I=512, qtype=2, codes=FAKE.value, scales=FAKE.value, hib=None):
    g = moe.QMat(qtype, E, I, H, codes, hib, scales)
    u = moe.QMat(qtype, E, I, H, codes, hib, scales)
    d = moe.QMat(qtype, E, H, I, codes, hib, scales)
    return moe.ExpertSet(g, u, d)


def _lf(lib, T=1, desc=None, routed=None, shared=None, x=FAKE, y=FAKE, ws=FAKE, wsb=1 << 40, path=0):
    desc = desc or _desc()
    routed = routed or _set()
    return lib.moe_layer_forward(x, T, FAKE, None, ctypes.byref(desc), ctypes.byref(routed),
                                 ctypes.byref(shared) if shared else None, None, y, None, None, path, ws,
                                 ctypes.c_size_t(wsb), None)


def test_layer_forward_validation(lib):
    assert _lf(lib, T=0) == moe.MOE_OK                                      # no-op
    assert _lf(lib, T=-1) == moe.MOE_ERR_INVALID_ARG
    assert _lf(lib, desc=_desc(H=100)) == moe.MOE_ERR_INVALID_ARG
    assert _lf(lib, desc=_desc(H=2016)) == moe.MOE_ERR_UNSUPPORTED         # multiple of 32, not of 64
    assert _lf(lib, desc=_desc(k=0)) == moe.MOE_ERR_INVALID_ARG
    assert _lf(lib, desc=_desc(k=513)) == moe.MOE_ERR_INVALID_ARG
    assert _lf(lib, desc=_desc(sh=1)) == moe.MOE_ERR_INVALID_ARG           # shared requested, none given
    assert _lf(lib, x=None) == moe.MOE_ERR_INVALID_ARG
    assert _lf(lib, x=FAKE_MIS) == moe.MOE_ERR_ALIGNMENT
    assert _lf(lib, routed=_set(codes=FAKE_MIS.value)) == moe.MOE_ERR_ALIGNMENT
    assert _lf(lib, routed=_set(qtype=3)) == moe.MOE_ERR_INVALID_ARG       # Q3 without the hi-bit plane
    assert _lf(lib, routed=_set(qtype=5)) == moe.MOE_ERR_INVALID_ARG
    assert _lf(lib, routed=_set(qtype=2, hib=FAKE.value)) == moe.MOE_ERR_INVALID_ARG  # hi bits belong to Q3 only
    assert _lf(lib, routed=_set(qtype=4, hib=FAKE.value)) == moe.MOE_ERR_INVALID_ARG
    assert _lf(lib, routed=_set(E=511)) == moe.MOE_ERR_INVALID_ARG         # set shape disagrees with desc
    # the shared expert in another block format than the routed experts (one format per layer)
    assert _lf(lib, desc=_desc(sh=1), shared=_set(E=1, qtype=4)) == moe.MOE_ERR_INVALID_ARG
    assert _lf(lib, ws=None) == moe.MOE_ERR_WORKSPACE
    assert _lf(lib, wsb=1024) == moe.MOE_ERR_WORKSPACE
    assert _lf(lib, path=5) == moe.MOE_ERR_INVALID_ARG
    assert _lf(lib, desc=_desc(H=2048, I=192), routed=_set(I=192), path=4) == moe.MOE_ERR_UNSUPPORTED  # mid: I % 128
    assert _lf(lib, T=129, path=4) == moe.MOE_ERR_UNSUPPORTED               # mid: at most 128 tokens
    assert _lf(lib, desc=_desc(H=2048, I=192), routed=_set(I=192), path=2) == moe.MOE_ERR_UNSUPPORTED


def test_router_permute_combine_validation(lib):
    sz = ctypes.c_size_t(1 << 40)
    assert lib.moe_router_topk(FAKE, 0, 2048, FAKE, None, 512, 10, FAKE, FAKE, None, FAKE, sz, None) == 0
    assert lib.moe_router_topk(FAKE, 4, 2048, FAKE, None, 512, 0, FAKE, FAKE, None, FAKE, sz, None) == 1
    assert lib.moe_router_topk(FAKE, 4, 2048, FAKE, None, 8, 9, FAKE, FAKE, None, FAKE, sz, None) == 1
    assert lib.moe_router_topk(FAKE, 4, 2048, FAKE, None, 5000, 9, FAKE, FAKE, None, FAKE, sz, None) == 1
    assert lib.moe_router_topk(FAKE_MIS, 4, 2048, FAKE, None, 512, 10, FAKE, FAKE, None, FAKE, sz, None) == 2
    assert lib.moe_router_topk(FAKE, 4, 2048, FAKE, None, 512, 10, FAKE, FAKE, None, FAKE, ctypes.c_size_t(64),
                               None) == 3
    assert lib.moe_permute(FAKE, 4, 10, 512, FAKE, 2048, 1, None, FAKE, FAKE, FAKE, FAKE, FAKE, sz, None) == 1
    assert lib.moe_combine(FAKE, FAKE, FAKE, 4, 0, 2048, None, None, FAKE, None) == 1
    assert lib.moe_combine(FAKE, FAKE, FAKE, 4, 10, 2048, None, None, FAKE_MIS, None) == 2
    assert lib.moe_combine(FAKE, FAKE, FAKE, 0, 10, 2048, None, None, FAKE, None) == 0
    rs = _set()
    assert lib.moe_expert_ffn(FAKE, FAKE, 10, 512, 2048, 512, ctypes.byref(rs), None, FAKE, 7, FAKE, sz, None) == 1
    assert lib.moe_expert_ffn(FAKE, FAKE, 0, 512, 2048, 512, ctypes.byref(rs), None, FAKE, 0, FAKE, sz, None) == 0
    assert lib.moe_rmsnorm_bf16(FAKE, 4, 2000, ctypes.c_float(1e-6), FAKE, None) == 1
    assert lib.moe_rmsnorm_bf16(FAKE, 4, 2048, ctypes.c_float(-1.0), FAKE, None) == 1
    q = moe.QMat(2, 4, 16, 64, FAKE.value, None, FAKE.value)
    assert lib.moe_dequant_rows(ctypes.byref(q), 4, 0, 1, FAKE, None, None) == 1   # expert out of range
    assert lib.moe_dequant_rows(ctypes.byref(q), 0, 10, 7, FAKE, None, None) == 1  # rows out of range
    assert lib.moe_dequant_rows(ctypes.byref(q), 0, 0, 1, None, None, None) == 1   # no output
    assert lib.moe_read_device_error(None, None, None) == 1
    assert lib.moe_workspace_init(None, ctypes.c_size_t(0), None) == 1
    assert lib.moe_workspace_init(FAKE, ctypes.c_size_t(16), None) == 3


def test_wait_timeout_hook_validation(lib):
    # host-side argument checks only; the timeout itself is exercised on the GPU
    assert lib.moe_test_wait_timeout(None, ctypes.c_size_t(1 << 20), 20, None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_test_wait_timeout(FAKE, ctypes.c_size_t(1024), 20, None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_test_wait_timeout(FAKE, ctypes.c_size_t(1 << 20), 0, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_test_wait_timeout(FAKE, ctypes.c_size_t(1 << 20), 5000, None) == moe.MOE_ERR_INVALID_ARG


def test_stack_validation(lib):
    d = _desc()
    assert lib.moe_stack_forward(FAKE, 4, 2, None, None, ctypes.byref(d), None, None, ctypes.c_float(1e-6), FAKE, 0,
                                 FAKE, ctypes.c_size_t(1 << 40), None) == 1
    assert lib.moe_stack_forward(FAKE, 4, -1, None, None, ctypes.byref(d), None, None, ctypes.c_float(1e-6), FAKE, 0,
                                 FAKE, ctypes.c_size_t(1 << 40), None) == 1


def _lfh(lib, T=1, desc=None, routed=None, x_host=FAKE, y_host=FAKE, ws=FAKE, wsb=1 << 40, path=0):
    desc = desc or _desc()
    routed = routed or _set()
    return lib.moe_layer_forward_host(x_host, T, FAKE, None, ctypes.byref(desc), ctypes.byref(routed), None, y_host,
                                      None, None, path, ws, ctypes.c_size_t(wsb), None)


def test_host_buffer_entry_points_validate_before_enqueueing(lib):
    # every rejection comes from the host checks that run before the first copy is enqueued
    assert _lfh(lib, T=0) == moe.MOE_OK
    assert _lfh(lib, T=-1) == moe.MOE_ERR_INVALID_ARG
    assert _lfh(lib, x_host=None) == moe.MOE_ERR_INVALID_ARG
    assert _lfh(lib, y_host=None) == moe.MOE_ERR_INVALID_ARG
    assert _lfh(lib, ws=None) == moe.MOE_ERR_WORKSPACE
    assert _lfh(lib, wsb=1024) == moe.MOE_ERR_WORKSPACE
    assert _lfh(lib, path=5) == moe.MOE_ERR_INVALID_ARG
    assert _lfh(lib, desc=_desc(H=2016)) == moe.MOE_ERR_UNSUPPORTED
    assert _lfh(lib, T=129, path=4) == moe.MOE_ERR_UNSUPPORTED
    assert _lfh(lib, routed=_set(qtype=3)) == moe.MOE_ERR_INVALID_ARG
    d = _desc()
    eps = ctypes.c_float(1e-6)
    assert lib.moe_stack_forward_host(None, 4, 2, None, None, ctypes.byref(d), None, None, eps, FAKE, 0, FAKE,
                                      ctypes.c_size_t(1 << 40), None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_stack_forward_host(FAKE, 4, 2, None, None, ctypes.byref(d), None, None, eps, FAKE, 0, FAKE,
                                      ctypes.c_size_t(1 << 40), None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_stack_forward_host(FAKE, 4, 2, None, None, ctypes.byref(d), None, None, eps, FAKE, 0, None,
                                      ctypes.c_size_t(1 << 40), None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_stack_forward_host(FAKE, 0, 2, None, None, ctypes.byref(d), None, None, eps, FAKE, 0, FAKE,
                                      ctypes.c_size_t(1 << 40), None) == moe.MOE_OK


def test_static_router_validation(lib):
    # host-side checks of the workspace-free router; none of these calls reaches the device
    def call(x=FAKE, T=1, H=2048, Wr=FAKE, E=512, k=10, idx=FAKE, w=FAKE):
        return lib.moe_router_topk_static(x, T, H, Wr, None, E, k, idx, w, None, None)
    assert call(H=100) == moe.MOE_ERR_INVALID_ARG        # H not a multiple of 64
    assert call(k=0) == moe.MOE_ERR_INVALID_ARG
    assert call(k=11, E=10) == moe.MOE_ERR_INVALID_ARG   # k > E
    assert call(T=-1) == moe.MOE_ERR_INVALID_ARG
    assert call(T=9) == moe.MOE_ERR_UNSUPPORTED           # beyond the fixed scratch
    assert call(T=0) == moe.MOE_OK                        # nothing to do
    assert call(x=None) == moe.MOE_ERR_INVALID_ARG
    assert call(x=FAKE_MIS) == moe.MOE_ERR_ALIGNMENT


def test_kernel_names_and_timing_queries(lib):
    n = lib.moe_kernel_count()
    names = [lib.moe_kernel_name(i) for i in range(n)]
    assert n > 0 and all(names) and len(set(names)) == n  # every kernel id has its own name
    assert lib.moe_kernel_name(n) is None and lib.moe_kernel_name(-1) is None
    ms, cnt = ctypes.c_double(0.0), ctypes.c_int32(0)
    assert lib.moe_timing_read(-1, ctypes.byref(ms), ctypes.byref(cnt)) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_timing_read(n, ctypes.byref(ms), ctypes.byref(cnt)) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_timing_read(0, None, ctypes.byref(cnt)) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_timing_enable(0) == moe.MOE_OK
    assert lib.moe_timing_read(0, ctypes.byref(ms), ctypes.byref(cnt)) == moe.MOE_OK
    assert cnt.value == 0 and ms.value == 0.0             # nothing was timed
