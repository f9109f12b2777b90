"""The C-ABI library loads, exports every symbol include/moe.h declares, and
rejects bad arguments before touching a GPU (runs on a CPU-only host)."""
import ctypes
import os
import re

import pytest

import mixture_experts_expert_softmax_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_\w+)\s*\(", text)))


def test_header_declares_the_exports():
    declared = header_functions()
    assert "moe_route" in declared and "moe_forward" in declared
    assert sorted(moe.EXPORTED) == declared


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(moe.LIB_PATH)
    for name in header_functions():
        assert hasattr(lib, name), name


def test_error_strings():
    for code in range(0, -8, -1):
        s = moe.error_string(code)
        assert s and "unknown" not in s
    assert "unknown" in moe.error_string(-99)


L = moe._lib
NULL = None


@pytest.mark.parametrize("args,code", [
    ((NULL, 4, 8, 2, 1, NULL, NULL, NULL), moe.MOE_ERR_INVALID_ARG),   # null pointers
    ((1, -1, 8, 2, 1, 1, 1, NULL), moe.MOE_ERR_INVALID_ARG),          # T < 0
    ((1, 4, 8, 9, 1, 1, 1, NULL), moe.MOE_ERR_INVALID_ARG),           # k > E
    ((1, 4, 8, 0, 1, 1, 1, NULL), moe.MOE_ERR_INVALID_ARG),           # k < 1
    ((1, 4, 0, 1, 1, 1, 1, NULL), moe.MOE_ERR_INVALID_ARG),           # E < 1
    ((1, 4, 2048, 2, 1, 1, 1, NULL), moe.MOE_ERR_UNSUPPORTED),        # E > 1024
    ((NULL, 0, 8, 2, 1, NULL, NULL, NULL), moe.MOE_OK),               # T == 0: nothing to do
])
def test_route_argument_checks(args, code):
    assert L.moe_route(*args) == code


# non-null stand-ins for device pointers, 16-byte aligned like real arrays
FWD_OK = dict(h=256, w1=256, w2=256, w=256, ids=256, out=256, T=4, H=256, I=128, E=8, k=2)


def fwd(**kw):
    a = dict(FWD_OK, **kw)
    return L.moe_forward(a["h"], a["w1"], a["w2"], a["w"], a["ids"], a["out"], a["T"], a["H"],
                         a["I"], a["E"], a["k"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(h=NULL), moe.MOE_ERR_INVALID_ARG),
    (dict(out=NULL), moe.MOE_ERR_INVALID_ARG),
    (dict(T=-1), moe.MOE_ERR_INVALID_ARG),
    (dict(k=9), moe.MOE_ERR_INVALID_ARG),
    (dict(k=0), moe.MOE_ERR_INVALID_ARG),
    (dict(H=0), moe.MOE_ERR_INVALID_ARG),
    (dict(H=200), moe.MOE_ERR_UNSUPPORTED),       # H % 128
    (dict(I=96), moe.MOE_ERR_UNSUPPORTED),        # I % 128
    (dict(E=2000, k=2), moe.MOE_ERR_UNSUPPORTED),  # E > 1024
    (dict(E=64, k=17), moe.MOE_ERR_UNSUPPORTED),   # k > 16
    (dict(T=0, h=NULL, out=NULL), moe.MOE_OK),    # empty batch
    (dict(h=264), moe.MOE_ERR_INVALID_ARG),        # hidden not 16-byte aligned
    (dict(w2=260), moe.MOE_ERR_INVALID_ARG),       # w2 not 16-byte aligned
    (dict(out=258), moe.MOE_ERR_INVALID_ARG),      # out not 16-byte aligned
])
def test_forward_argument_checks(kw, code):
    assert fwd(**kw) == code


def fwd_ex(b1=NULL, b2=NULL, act=0, **kw):
    a = dict(FWD_OK, **kw)
    return L.moe_forward_ex(a["h"], a["w1"], a["w2"], b1, b2, act, a["w"], a["ids"], a["out"],
                            a["T"], a["H"], a["I"], a["E"], a["k"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(act=3), moe.MOE_ERR_INVALID_ARG),         # unknown activation
    (dict(act=-1), moe.MOE_ERR_INVALID_ARG),
    (dict(b1=260), moe.MOE_ERR_INVALID_ARG),        # b1 not 16-byte aligned
    (dict(b2=264, act=2), moe.MOE_ERR_INVALID_ARG),  # b2 not 16-byte aligned
    (dict(act=1, H=200), moe.MOE_ERR_UNSUPPORTED),
    (dict(act=2, h=NULL), moe.MOE_ERR_INVALID_ARG),
    (dict(act=1, T=0, h=NULL, out=NULL), moe.MOE_OK),
])
def test_forward_ex_argument_checks(kw, code):
    assert fwd_ex(**kw) == code


def fwd_fp8(s1=256, s2=256, block=128, **kw):
    a = dict(FWD_OK, **kw)
    return L.moe_forward_fp8(a["h"], a["w1"], s1, a["w2"], s2, block, a["w"], a["ids"], a["out"],
                             a["T"], a["H"], a["I"], a["E"], a["k"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(s1=NULL), moe.MOE_ERR_INVALID_ARG),      # scales missing
    (dict(s2=NULL), moe.MOE_ERR_INVALID_ARG),
    (dict(block=0), moe.MOE_ERR_INVALID_ARG),
    (dict(block=64), moe.MOE_ERR_UNSUPPORTED),     # not a multiple of 128
    (dict(block=256, I=128), moe.MOE_ERR_UNSUPPORTED),  # does not divide I
    (dict(w1=260), moe.MOE_ERR_INVALID_ARG),       # codes not 16-byte aligned
    (dict(T=0, h=NULL, out=NULL), moe.MOE_OK),
])
def test_forward_fp8_argument_checks(kw, code):
    assert fwd_fp8(**kw) == code


def test_binding_rejects_unknown_activation():
    import torch
    t = torch.empty(0)
    with pytest.raises(ValueError, match="act must be one of"):
        moe.moe_forward(t, t, t, t, t, act="relu")


def test_permute_argument_checks():
    assert L.moe_permute(NULL, 4, 2, 8, NULL, NULL, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_permute(1, 4, 0, 8, 1, 1, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_permute(1, 4, 2, 4096, 1, 1, None) == moe.MOE_ERR_UNSUPPORTED


def perm_ex(ids=256, T=4, k=2, E=8, rows=256, offs=256, inv=NULL, h=NULL, H=0, xs=NULL,
            kernel=0):
    return L.moe_permute_ex(ids, T, k, E, rows, offs, inv, h, H, xs, kernel, None)


@pytest.mark.parametrize("kw,code", [
    (dict(ids=NULL), moe.MOE_ERR_INVALID_ARG),
    (dict(offs=NULL), moe.MOE_ERR_INVALID_ARG),
    (dict(kernel=3), moe.MOE_ERR_INVALID_ARG),           # unknown grouping kernel
    (dict(h=256, H=256), moe.MOE_ERR_INVALID_ARG),        # hidden without xs
    (dict(xs=256, H=256), moe.MOE_ERR_INVALID_ARG),       # xs without hidden
    (dict(h=264, xs=256, H=256), moe.MOE_ERR_INVALID_ARG),  # hidden not 16-byte aligned
    (dict(h=256, xs=256, H=0), moe.MOE_ERR_INVALID_ARG),
    (dict(h=256, xs=256, H=200), moe.MOE_ERR_UNSUPPORTED),  # H % 128
    (dict(E=2000), moe.MOE_ERR_UNSUPPORTED),
    (dict(T=4097, k=2, kernel=1), moe.MOE_ERR_UNSUPPORTED),  # > 8192 entries, one kernel
])
def test_permute_ex_argument_checks(kw, code):
    assert perm_ex(**kw) == code


def test_timeline_argument_checks():
    assert L.moe_timeline(256, 0) == moe.MOE_ERR_INVALID_ARG    # capacity < 1
    assert L.moe_timeline(260, 16) == moe.MOE_ERR_INVALID_ARG   # not 8-byte aligned
    assert L.moe_timeline(256, 16) == moe.MOE_OK                # set (no device access)
    assert L.moe_timeline(None, 0) == moe.MOE_OK                # off


def test_ep_argument_checks():
    i64 = ctypes.c_int64
    offs = (i64 * 3)(0, 2, 5)
    row0 = (i64 * 2)(0, 0)
    ptrs = (ctypes.c_void_p * 2)(256, 256)
    # dispatch plan
    assert L.moe_ep_dispatch_plan(256, 4, 2, 8, 0, 256, 256, 256, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_ep_dispatch_plan(256, 4, 2, 8, 3, 256, 256, 256, None) == moe.MOE_ERR_UNSUPPORTED
    assert L.moe_ep_dispatch_plan(256, 4, 2, 8, 65, 256, 256, 256, None) == moe.MOE_ERR_UNSUPPORTED
    assert L.moe_ep_dispatch_plan(NULL, 4, 2, 8, 2, 256, 256, 256, None) == moe.MOE_ERR_INVALID_ARG
    # pack: offsets must be a prefix sum from 0 within T*k
    assert L.moe_ep_pack(256, 256, 256, 4, 2, 8, 2, 256, offs, ptrs, ptrs, row0,
                         None) in (moe.MOE_ERR_NO_DEVICE, moe.MOE_OK)
    bad = (i64 * 3)(1, 2, 5)
    assert L.moe_ep_pack(256, 256, 256, 4, 2, 8, 2, 256, bad, ptrs, ptrs, row0,
                         None) == moe.MOE_ERR_INVALID_ARG
    down = (i64 * 3)(0, 4, 3)
    assert L.moe_ep_pack(256, 256, 256, 4, 2, 8, 2, 256, down, ptrs, ptrs, row0,
                         None) == moe.MOE_ERR_INVALID_ARG
    big = (i64 * 3)(0, 4, 9)  # more rows than T*k
    assert L.moe_ep_pack(256, 256, 256, 4, 2, 8, 2, 256, big, ptrs, ptrs, row0,
                         None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_ep_pack(256, 200, 256, 4, 2, 8, 2, 256, offs, ptrs, ptrs, row0,
                         None) == moe.MOE_ERR_UNSUPPORTED
    # return and combine
    assert L.moe_ep_return(256, 256, 2, bad, ptrs, row0, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_ep_return(264, 256, 2, offs, ptrs, row0, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_ep_combine(256, 256, 256, 256, 4, 200, 2, None) == moe.MOE_ERR_UNSUPPORTED
    assert L.moe_ep_combine(NULL, 256, 256, 256, 4, 256, 2, None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_ep_combine(NULL, NULL, NULL, NULL, 0, 256, 2, None) == moe.MOE_OK


def test_debug_switches_roundtrip():
    prev = moe.set_small_t_max(5)
    assert moe.set_small_t_max(prev) == 5
    prev = moe.set_sync_each_stage(True)
    assert moe.set_sync_each_stage(prev) == 1
    prev = moe.set_wait_limit_ns(12345)
    assert moe.set_wait_limit_ns(prev) == 12345
    assert moe.debug_wait_timeout(0) == moe.MOE_ERR_INVALID_ARG


def test_no_gpu_fails_loudly():
    """Without a usable sm_100 device the library reports it; it never falls back."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert L.moe_route(1, 4, 8, 2, 1, 1, 1, None) == moe.MOE_ERR_NO_DEVICE
    assert fwd() == moe.MOE_ERR_NO_DEVICE
    assert fwd_ex(act=1, b1=256, b2=256) == moe.MOE_ERR_NO_DEVICE
    assert fwd_fp8() == moe.MOE_ERR_NO_DEVICE
