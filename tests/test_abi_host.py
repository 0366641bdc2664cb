"""The C-ABI library on the host: it loads, exports exactly what include/wf.h declares, and its
argument validation answers before anything touches a GPU."""
import ctypes
import os
import re

import pytest
import torch

from block_causal_streaming_b200 import build as wf_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wf.h")


@pytest.fixture(scope="module")
def abi():
    wf_build.build()
    from block_causal_streaming_b200 import _abi
    return _abi


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(wf_\w+)\s*\(", text, re.M)))


def test_header_declarations_match_binding(abi):
    assert declared_functions() == sorted(abi.EXPORTED)


def test_library_exports_every_declared_symbol(abi):
    lib = ctypes.CDLL(abi.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} is declared but not exported"


def test_header_error_codes_match_binding(abi):
    text = open(HEADER).read()
    codes = dict((m.group(1), int(m.group(2)))
                 for m in re.finditer(r"(WF_(?:OK|ERR_\w+))\s*=\s*(\d+)", text))
    for name, value in codes.items():
        assert getattr(abi, name) == value, name
    assert abi.WF_MAX_CHUNKS == int(re.search(r"#define WF_MAX_CHUNKS (\d+)", text).group(1))


def test_strerror_and_version(abi):
    for code in range(0, 9):
        assert abi.strerror(code).startswith("WF_")
    assert "unknown" in abi.strerror(99)
    assert abi.lib.wf_version() >= 100


FAKE = 0x10000  # an aligned, never-dereferenced address: validation must answer first


def _pool(abi, **kw):
    args = dict(k_pool=FAKE, v_pool=FAKE, num_pages=8, page_size=64, num_heads=2, head_dim=128)
    args.update(kw)
    return abi.KvPool(**args)


def _attn(abi, pool, desc, scale=0.1, q=FAKE, out=FAKE, pt=FAKE):
    return abi.lib.wf_attn_forward(q, ctypes.byref(pool),
                                   ctypes.cast(ctypes.c_void_p(pt), ctypes.POINTER(ctypes.c_int32)),
                                   ctypes.byref(desc.c), scale, out, None, None)


def _append(abi, pool, desc, layer=0, chunk=0, k=FAKE, v=FAKE, pt=FAKE):
    return abi.lib.wf_kv_append(ctypes.byref(pool), layer, chunk, k, v,
                                ctypes.cast(ctypes.c_void_p(pt), ctypes.POINTER(ctypes.c_int32)),
                                ctypes.byref(desc.c), None)


def test_validation_errors_without_a_gpu(abi):
    ok_desc = abi.WavefrontDesc([0, 64, 128, 200], [0, 200, 1000], 1, 8)
    # pool checks
    assert _attn(abi, _pool(abi, k_pool=0), ok_desc) == abi.WF_ERR_INVALID_ARG
    assert _attn(abi, _pool(abi, v_pool=FAKE + 8), ok_desc) == abi.WF_ERR_INVALID_ARG
    assert _attn(abi, _pool(abi, head_dim=96), ok_desc) == abi.WF_ERR_SHAPE
    assert _attn(abi, _pool(abi, page_size=24), ok_desc) == abi.WF_ERR_SHAPE
    assert _attn(abi, _pool(abi, page_size=0), ok_desc) == abi.WF_ERR_SHAPE
    assert _attn(abi, _pool(abi, num_heads=0), ok_desc) == abi.WF_ERR_SHAPE
    # descriptor checks
    assert _attn(abi, _pool(abi), abi.WavefrontDesc([1, 64, 128], [0, 0], 0, 8)) == \
        abi.WF_ERR_SHAPE
    assert _attn(abi, _pool(abi), abi.WavefrontDesc([0, 64, 60], [0, 0], 0, 8)) == \
        abi.WF_ERR_SHAPE
    assert _attn(abi, _pool(abi), abi.WavefrontDesc([0, 64, 128], [500, 200], 0, 8)) == \
        abi.WF_ERR_STAGE_ORDER
    assert _attn(abi, _pool(abi), abi.WavefrontDesc([0, 64, 600], [0, 0], 0, 8)) == \
        abi.WF_ERR_CAPACITY
    assert _attn(abi, _pool(abi), abi.WavefrontDesc([0, 64, 128], [0, 0], 2, 8)) == \
        abi.WF_ERR_SHAPE                                          # no query chunk
    too_many = list(range(0, 66))
    assert _attn(abi, _pool(abi), abi.WavefrontDesc(too_many, [0] * 65, 0, 8)) == \
        abi.WF_ERR_SHAPE
    # call arguments
    assert _attn(abi, _pool(abi), ok_desc, scale=0.0) == abi.WF_ERR_INVALID_ARG
    assert _attn(abi, _pool(abi), ok_desc, scale=float("nan")) == abi.WF_ERR_INVALID_ARG
    assert _attn(abi, _pool(abi), ok_desc, q=0) == abi.WF_ERR_INVALID_ARG
    assert _attn(abi, _pool(abi), ok_desc, out=FAKE + 2) == abi.WF_ERR_INVALID_ARG
    assert _append(abi, _pool(abi), ok_desc, chunk=3) == abi.WF_ERR_INVALID_ARG
    assert _append(abi, _pool(abi), ok_desc, layer=-1) == abi.WF_ERR_INVALID_ARG
    assert _append(abi, _pool(abi), ok_desc, k=FAKE + 4) == abi.WF_ERR_INVALID_ARG


def test_selftest_timeout_rejects_bad_limits(abi):
    assert abi.lib.wf_selftest_timeout(0, None) == abi.WF_ERR_INVALID_ARG
    assert abi.lib.wf_selftest_timeout(2000000, None) == abi.WF_ERR_INVALID_ARG


def test_empty_work_is_a_no_op(abi):
    """T_q = 0 and empty chunks return WF_OK before any device work."""
    desc = abi.WavefrontDesc([0, 64, 64], [0, 0], 1, 8)        # the only query chunk is empty
    assert _attn(abi, _pool(abi), desc) == abi.WF_OK
    assert _append(abi, _pool(abi), desc, chunk=1) == abi.WF_OK


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device answer")
def test_valid_call_without_device_reports_no_device(abi):
    desc = abi.WavefrontDesc([0, 64, 128, 200], [0, 200, 1000], 1, 8)
    assert _attn(abi, _pool(abi), desc) == abi.WF_ERR_NO_DEVICE
    assert _append(abi, _pool(abi), desc) == abi.WF_ERR_NO_DEVICE


def test_split_workspace_size_formula(abi):
    """S * T_q * H * (D + 1) fp32 values, each array rounded up to 256 bytes; none for S = 1."""
    desc = abi.WavefrontDesc([0, 4680, 9360], [0, 1000], 1, 200)     # T_q = 4680
    for heads, d, s in ((12, 128, 4), (2, 64, 3), (40, 128, 16)):
        rows = s * 4680 * heads
        up = lambda n: (n + 255) // 256 * 256
        assert abi.lib.wf_attn_workspace_size(ctypes.byref(desc.c), heads, d, s) == \
            up(rows * d * 4) + up(rows * 4)
    assert abi.lib.wf_attn_workspace_size(ctypes.byref(desc.c), 12, 128, 1) == 0
    # capped at the key tiles of the smallest unit: 9360 keys = 74 tiles, cap 16
    assert abi.lib.wf_attn_workspace_size(ctypes.byref(desc.c), 12, 128, 99) == \
        abi.lib.wf_attn_workspace_size(ctypes.byref(desc.c), 12, 128, 16)
    small = abi.WavefrontDesc([0, 100, 200], [0, 0], 1, 200)        # 200 keys: 2 tiles
    assert abi.lib.wf_attn_workspace_size(ctypes.byref(small.c), 1, 128, 8) == \
        abi.lib.wf_attn_workspace_size(ctypes.byref(small.c), 1, 128, 2)
    # invalid arguments give 0 (the forward call reports the error)
    assert abi.lib.wf_attn_workspace_size(ctypes.byref(desc.c), 12, 96, 4) == 0
    assert abi.lib.wf_attn_workspace_size(ctypes.byref(desc.c), 0, 128, 4) == 0
    assert abi.lib.wf_attn_workspace_size(ctypes.byref(desc.c), 12, 128, -1) == 0


def test_split_validation_errors_without_a_gpu(abi):
    ok_desc = abi.WavefrontDesc([0, 64, 128, 200], [0, 200, 1000], 1, 8)

    def split(pool, desc, splits=2, ws=None, nbytes=0):
        return abi.lib.wf_attn_forward_split(
            FAKE, ctypes.byref(pool), ctypes.cast(ctypes.c_void_p(FAKE), ctypes.POINTER(ctypes.c_int32)),
            ctypes.byref(desc.c), 0.1, FAKE, None, splits, ws, nbytes, None)
    assert split(_pool(abi), ok_desc, splits=-1) == abi.WF_ERR_INVALID_ARG
    assert split(_pool(abi, head_dim=96), ok_desc) == abi.WF_ERR_SHAPE
    assert split(_pool(abi), abi.WavefrontDesc([0, 64, 128], [500, 200], 0, 8)) == \
        abi.WF_ERR_STAGE_ORDER
    empty = abi.WavefrontDesc([0, 64, 64], [0, 0], 1, 8)
    assert split(_pool(abi), empty) == abi.WF_OK


def _fp8_pool(abi, **kw):
    args = dict(k_codes=FAKE, v_codes=FAKE, k_scale=FAKE, v_scale=FAKE, num_pages=8, page_size=64,
                num_heads=2, head_dim=128)
    args.update(kw)
    return abi.KvPoolFp8(**args)


def test_fp8_validation_errors_without_a_gpu(abi):
    desc = abi.WavefrontDesc([0, 64, 128, 200], [0, 200, 1000], 1, 8)
    pt = ctypes.cast(ctypes.c_void_p(FAKE), ctypes.POINTER(ctypes.c_int32))

    def append(pool, chunk=0, k=FAKE):
        return abi.lib.wf_kv_append_fp8(ctypes.byref(pool), 0, chunk, k, FAKE, pt,
                                        ctypes.byref(desc.c), None)

    def dequant(src, dst, chunk=0):
        return abi.lib.wf_kv_dequant(ctypes.byref(src), ctypes.byref(dst), 0, chunk, pt,
                                     ctypes.byref(desc.c), None)
    assert append(_fp8_pool(abi, k_scale=FAKE + 4)) == abi.WF_ERR_INVALID_ARG    # misaligned
    assert append(_fp8_pool(abi, v_codes=None)) == abi.WF_ERR_INVALID_ARG
    assert append(_fp8_pool(abi, head_dim=96)) == abi.WF_ERR_SHAPE
    assert append(_fp8_pool(abi, page_size=24)) == abi.WF_ERR_SHAPE
    assert append(_fp8_pool(abi), chunk=3) == abi.WF_ERR_INVALID_ARG             # no such chunk
    assert append(_fp8_pool(abi), k=FAKE + 2) == abi.WF_ERR_INVALID_ARG
    short = abi.WavefrontDesc([0, 64, 128, 200], [0, 200, 1000], 1, 2)   # 4 pages needed > 2
    assert abi.lib.wf_kv_append_fp8(ctypes.byref(_fp8_pool(abi)), 0, 0, FAKE, FAKE, pt,
                                    ctypes.byref(short.c), None) == abi.WF_ERR_CAPACITY
    assert dequant(_fp8_pool(abi), _pool(abi, num_heads=3)) == abi.WF_ERR_SHAPE  # geometries differ
    assert dequant(_fp8_pool(abi), _pool(abi, k_pool=FAKE + 8)) == abi.WF_ERR_INVALID_ARG
    empty = abi.WavefrontDesc([0, 64, 64], [0, 0], 1, 8)
    assert abi.lib.wf_kv_append_fp8(ctypes.byref(_fp8_pool(abi)), 0, 1, FAKE, FAKE, pt,
                                    ctypes.byref(empty.c), None) == abi.WF_OK      # empty chunk
    if not torch.cuda.is_available():
        assert append(_fp8_pool(abi)) == abi.WF_ERR_NO_DEVICE
        assert dequant(_fp8_pool(abi), _pool(abi)) == abi.WF_ERR_NO_DEVICE


def _qk(abi, e4m3, **kw):
    fields = abi.QK_E4M3_FIELDS if e4m3 else abi.QK_I8_FIELDS
    args = {n: FAKE for n in fields}
    args.update(kw)
    return (abi.QkE4m3 if e4m3 else abi.QkI8)(**args)


@pytest.mark.parametrize("e4m3", [False, True], ids=["int8", "e4m3"])
def test_8bit_tier_validation_errors_without_a_gpu(abi, e4m3):
    """The INT8 / FP8 attention tiers answer bad arguments, and empty work, before any device
    work; a valid call on a machine without a GPU reports WF_ERR_NO_DEVICE."""
    desc = abi.WavefrontDesc([0, 64, 128, 200], [0, 200, 1000], 1, 8)
    empty = abi.WavefrontDesc([0, 64, 64], [0, 0], 1, 8)
    tier = "e4m3" if e4m3 else "i8"
    pt = ctypes.cast(ctypes.c_void_p(FAKE), ctypes.POINTER(ctypes.c_int32))

    def quantize(qk, pool=None, wf=desc, q=FAKE):
        return getattr(abi.lib, f"wf_qk_quantize_{tier}")(
            q, ctypes.byref(pool or _pool(abi)), pt, ctypes.byref(wf.c),
            ctypes.byref(qk) if qk is not None else None, None)

    def forward(qk, pool=None, wf=desc):
        return getattr(abi.lib, f"wf_attn_forward_{tier}")(
            ctypes.byref(qk) if qk is not None else None, ctypes.byref(pool or _pool(abi)), pt,
            ctypes.byref(wf.c), 0.1, FAKE, None, None)

    ok = _qk(abi, e4m3)
    assert quantize(None) == abi.WF_ERR_INVALID_ARG
    assert quantize(ok, q=FAKE + 8) == abi.WF_ERR_INVALID_ARG                  # q unaligned
    assert quantize(_qk(abi, e4m3, q_codes=FAKE + 8)) == abi.WF_ERR_INVALID_ARG
    assert quantize(_qk(abi, e4m3, k_scale=FAKE + 2)) == abi.WF_ERR_INVALID_ARG
    assert quantize(ok, pool=_pool(abi, head_dim=64)) == abi.WF_ERR_SHAPE
    assert quantize(ok, wf=empty) == abi.WF_OK                                 # no query rows
    assert forward(None) == abi.WF_ERR_INVALID_ARG
    assert forward(_qk(abi, e4m3, k_codes=FAKE + 8)) == abi.WF_ERR_INVALID_ARG
    assert forward(_qk(abi, e4m3, q_scale=None)) == abi.WF_ERR_INVALID_ARG
    assert forward(_qk(abi, e4m3, q_codes=FAKE + 8)) == abi.WF_ERR_INVALID_ARG
    assert forward(ok, pool=_pool(abi, head_dim=64)) == abi.WF_ERR_SHAPE
    assert forward(ok, wf=empty) == abi.WF_OK
    if not e4m3:
        assert quantize(_qk(abi, e4m3, k_sum=FAKE + 4)) == abi.WF_ERR_INVALID_ARG  # fp64
        assert quantize(_qk(abi, e4m3, k_mean=None)) == abi.WF_ERR_INVALID_ARG
    if not torch.cuda.is_available():
        assert quantize(ok) == abi.WF_ERR_NO_DEVICE
        assert forward(ok) == abi.WF_ERR_NO_DEVICE


def test_fp8_range_validation_errors_without_a_gpu(abi):
    """The chunk-range forms of the FP8 append and conversion: the range [begin, end) must be
    non-empty and inside the wavefront; empty chunks are no work."""
    desc = abi.WavefrontDesc([0, 64, 128, 200], [0, 200, 1000], 1, 8)
    pt = ctypes.cast(ctypes.c_void_p(FAKE), ctypes.POINTER(ctypes.c_int32))

    def append(begin, end, k=FAKE, wf=desc):
        return abi.lib.wf_kv_append_fp8_chunks(ctypes.byref(_fp8_pool(abi)), 0, begin, end, k,
                                               FAKE, pt, ctypes.byref(wf.c), None)

    def dequant(begin, end, dst=None):
        return abi.lib.wf_kv_dequant_chunks(ctypes.byref(_fp8_pool(abi)),
                                            ctypes.byref(dst or _pool(abi)), 0, begin, end, pt,
                                            ctypes.byref(desc.c), None)
    for begin, end in ((1, 1), (2, 1), (-1, 2), (0, 4)):
        assert append(begin, end) == abi.WF_ERR_INVALID_ARG
        assert dequant(begin, end) == abi.WF_ERR_INVALID_ARG
    assert append(0, 3, k=FAKE + 2) == abi.WF_ERR_INVALID_ARG
    assert dequant(0, 3, dst=_pool(abi, num_heads=3)) == abi.WF_ERR_SHAPE
    empty = abi.WavefrontDesc([0, 64, 64, 64], [0, 0, 0], 1, 8)
    assert append(1, 3, wf=empty) == abi.WF_OK                                  # no rows
    if not torch.cuda.is_available():
        assert append(0, 3) == abi.WF_ERR_NO_DEVICE
        assert dequant(1, 3) == abi.WF_ERR_NO_DEVICE
