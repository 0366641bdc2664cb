"""The binding's shape checks, on the CPU.

The C ABI takes plain pointers, so a tensor of the wrong shape would be read or written past its
end on the device.  The binding checks every shape against the descriptor and the pool geometry
first.  Here the library calls are replaced by a stand-in that answers WF_OK, and the CUDA-device
requirement is lifted, so the binding runs on CPU tensors.  Every call pattern the package's own
helpers make must pass, and malformed arguments must raise ValueError before anything is launched.
"""
import pytest
import torch

from block_causal_streaming_b200 import build as wf_build

wf_build.build()
from block_causal_streaming_b200 import _abi  # noqa: E402
from block_causal_streaming_b200.layer import PagedPool, PagedPoolFp8, WavefrontLayer  # noqa
from block_causal_streaming_b200.window import RollingCache, RollingWindow  # noqa: E402


class _FakeLib:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def call(*args):
            self.calls.append(name)
            return 0
        return call


@pytest.fixture
def fake(monkeypatch):
    lib = _FakeLib()
    real_check = _abi._check_tensor

    def check_on_cpu(t, name, dtype_name):
        if t.is_cuda:
            return real_check(t, name, dtype_name)
        if not t.is_contiguous():
            raise ValueError(f"{name}: expected a contiguous tensor")

    monkeypatch.setattr(_abi, "lib", lib)
    monkeypatch.setattr(_abi, "_check_tensor", check_on_cpu)
    monkeypatch.setattr(_abi, "_stream_handle", lambda s: None)
    return lib


H, D, PS = 2, 64, 16
OFF = [0, 40, 90, 130]          # one context chunk, two query chunks
STAGE = [0, 200, 1000]


def _layer(pages=10, layers=1):
    pool = PagedPool(pages * layers, PS, H, D, "cpu")
    pt = torch.arange(pages * layers, dtype=torch.int32).view(layers, pages)
    return WavefrontLayer(pool, pt, layers - 1, OFF, STAGE, 1)


def _kv(rows):
    return torch.zeros(rows, H, D, dtype=torch.bfloat16)


def test_the_helpers_valid_calls_pass(fake):
    lay = _layer()
    lay.append_range(_kv(130), _kv(130), range(3))
    q = _kv(90)
    out = torch.empty_like(q)
    lse = torch.empty(H, 90)
    lay.forward(q, out, lse=lse)
    lay.forward(q, out, splits=0)                     # workspace size comes back 0 from the fake
    fp = PagedPoolFp8(10, PS, H, D, "cpu")
    for c in range(3):
        _abi.kv_append_fp8(*fp.tensors, 0, c, _kv(OFF[c + 1] - OFF[c]), _kv(OFF[c + 1] - OFF[c]),
                           lay.page_tables, lay.desc)
        _abi.kv_dequant(*fp.tensors, lay.pool.k, lay.pool.v, 0, c, lay.page_tables, lay.desc)
    _abi.kv_append_fp8_chunks(*fp.tensors, 0, 0, 3, _kv(130), _kv(130), lay.page_tables, lay.desc)
    _abi.kv_append_fp8_chunks(*fp.tensors, 0, 1, 3, _kv(90), _kv(90), lay.page_tables, lay.desc)
    _abi.kv_dequant_chunks(*fp.tensors, lay.pool.k, lay.pool.v, 0, 0, 3, lay.page_tables,
                           lay.desc)
    flags = torch.zeros(2, _abi.WF_MAX_CHUNKS, dtype=torch.int32)
    _abi.kv_append_publish_fp8(*fp.tensors, flags, [], 0, 1, _kv(50), _kv(50), lay.page_tables,
                               lay.desc, 2)
    _abi.kv_dequant_published(*fp.tensors, lay.pool.k, lay.pool.v, 0, 1, lay.page_tables,
                              lay.desc, flags[0], 2)
    pt2 = torch.stack([lay.page_tables[0], lay.page_tables[0]]).contiguous()
    _abi.kv_append_publish(lay.pool.k, lay.pool.v, flags, [], 1, 2, _kv(40), _kv(40), pt2,
                           lay.desc, 3)
    _abi.attn_forward_published(q, lay.pool.k, lay.pool.v, pt2[1], lay.desc, 0.1, out, flags[1],
                                3)
    _abi.attn_forward_split_noalloc(q, lay.pool.k, lay.pool.v, lay.page_tables[0], lay.desc, 0.1,
                                    out)
    win = RollingWindow(24, [1000, 500], 2, 16)
    cache = RollingCache(win, H, D, 2, "cpu")
    for t in range(8):
        v = win.view(t)
        rows = v.t_q
        for layer in range(2):
            cache.run_layer(v, layer, _kv(rows), _kv(rows), _kv(rows), _kv(rows))
    assert "wf_attn_forward" in fake.calls and "wf_kv_dequant" in fake.calls
    for name in ("wf_kv_append_fp8_chunks", "wf_kv_dequant_chunks", "wf_kv_append_publish_fp8",
                 "wf_kv_dequant_published"):
        assert name in fake.calls


@pytest.mark.parametrize("case", [
    "k_rows", "v_shape", "k_heads", "pt_1d", "pt_width", "layer_out", "q_rows", "q_dim", "out",
    "lse_transposed", "row_short", "pool_mismatch", "fp8_scale", "dequant_geometry",
    "flags_small", "flags_row_small", "range_rows", "range_dequant_geometry",
    "fp8_publish_rows", "fp8_publish_flags_small", "fp8_dequant_flags_row_small",
])
def test_malformed_arguments_raise_before_any_launch(fake, case):
    lay = _layer()
    k, v, q = _kv(40), _kv(40), _kv(90)
    out, pt, row = torch.empty_like(q), lay.page_tables, lay.page_tables[0]
    fp = PagedPoolFp8(10, PS, H, D, "cpu")
    flags = torch.zeros(1, _abi.WF_MAX_CHUNKS, dtype=torch.int32)
    calls = {
        "k_rows": lambda: _abi.kv_append(lay.pool.k, lay.pool.v, 0, 0, _kv(39), v, pt, lay.desc),
        "v_shape": lambda: _abi.kv_append(lay.pool.k, lay.pool.v, 0, 0, k, _kv(41), pt, lay.desc),
        "k_heads": lambda: _abi.kv_append(lay.pool.k, lay.pool.v, 0, 0,
                                          torch.zeros(40, H + 1, D, dtype=torch.bfloat16), v, pt,
                                          lay.desc),
        "pt_1d": lambda: _abi.kv_append(lay.pool.k, lay.pool.v, 0, 0, k, v, row, lay.desc),
        "pt_width": lambda: _abi.kv_append(lay.pool.k, lay.pool.v, 0, 0, k, v,
                                           pt[:, :5].contiguous(), lay.desc),
        "layer_out": lambda: _abi.kv_append(lay.pool.k, lay.pool.v, 1, 0, k, v, pt, lay.desc),
        "q_rows": lambda: _abi.attn_forward(_kv(89), lay.pool.k, lay.pool.v, row, lay.desc, 0.1,
                                            _kv(89)),
        "q_dim": lambda: _abi.attn_forward(torch.zeros(90, H, 2 * D, dtype=torch.bfloat16),
                                           lay.pool.k, lay.pool.v, row, lay.desc, 0.1, out),
        "out": lambda: _abi.attn_forward(q, lay.pool.k, lay.pool.v, row, lay.desc, 0.1, _kv(91)),
        "lse_transposed": lambda: _abi.attn_forward(q, lay.pool.k, lay.pool.v, row, lay.desc, 0.1,
                                                    out, lse=torch.empty(90, H)),
        "row_short": lambda: _abi.attn_forward(q, lay.pool.k, lay.pool.v, row[:4].contiguous(),
                                               lay.desc, 0.1, out),
        "pool_mismatch": lambda: _abi.attn_forward(q, lay.pool.k, lay.pool.v[:5].contiguous(), row,
                                                   lay.desc, 0.1, out),
        "fp8_scale": lambda: _abi.kv_append_fp8(fp.k_codes, fp.v_codes, fp.k_scale[:, :8],
                                                fp.v_scale, 0, 0, k, v, pt, lay.desc),
        "dequant_geometry": lambda: _abi.kv_dequant(*fp.tensors, lay.pool.k[:9].contiguous(),
                                                    lay.pool.v[:9].contiguous(), 0, 0, pt,
                                                    lay.desc),
        "flags_small": lambda: _abi.kv_append_publish(lay.pool.k, lay.pool.v,
                                                      flags[:, :2].contiguous(), [], 0, 0, k, v,
                                                      pt, lay.desc, 1),
        "flags_row_small": lambda: _abi.attn_forward_published(
            q, lay.pool.k, lay.pool.v, row, lay.desc, 0.1, out, flags[0, :2].contiguous(), 1),
        # chunks [1, 3) hold 90 rows, not 130
        "range_rows": lambda: _abi.kv_append_fp8_chunks(*fp.tensors, 0, 1, 3, _kv(130), _kv(130),
                                                        pt, lay.desc),
        "range_dequant_geometry": lambda: _abi.kv_dequant_chunks(
            *fp.tensors, lay.pool.k[:9].contiguous(), lay.pool.v[:9].contiguous(), 0, 0, 3, pt,
            lay.desc),
        "fp8_publish_rows": lambda: _abi.kv_append_publish_fp8(*fp.tensors, flags, [], 0, 1,
                                                               _kv(40), _kv(40), pt, lay.desc, 1),
        "fp8_publish_flags_small": lambda: _abi.kv_append_publish_fp8(
            *fp.tensors, flags[:, :2].contiguous(), [], 0, 0, k, v, pt, lay.desc, 1),
        "fp8_dequant_flags_row_small": lambda: _abi.kv_dequant_published(
            *fp.tensors, lay.pool.k, lay.pool.v, 0, 0, pt, lay.desc, flags[0, :2].contiguous(), 1),
    }
    with pytest.raises(ValueError):
        calls[case]()
    assert fake.calls == []
