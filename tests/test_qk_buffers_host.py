"""The 8-bit attention tiers' buffers on the host: the library's sizes calls give the byte counts
of the layouts include/wf.h states, and the binding refuses buffers smaller than those before
anything reaches a GPU (the C ABI takes plain pointers and cannot see a buffer's size)."""
import pytest
import torch

from block_causal_streaming_b200 import build as wf_build

H, D = 2, 128
OFFSETS = [0, 64, 128, 200]          # one context chunk of 64 keys, query chunks of 64 and 72
T_KV, T_Q = 200, 136


@pytest.fixture(scope="module")
def abi():
    wf_build.build()
    from block_causal_streaming_b200 import _abi
    return _abi


def _desc(abi):
    return abi.WavefrontDesc(OFFSETS, [0, 200, 1000], 1, 8)


def _expected_i8():
    q_blocks, k_blocks = -(-T_Q // 128), -(-T_KV // 128)
    return [T_Q * H * D,                 # q_codes: one byte per element
            4 * H * q_blocks,            # q_scale: fp32 per (128 query rows, head)
            T_KV * H * D,                # k_codes, logical key order
            4 * H * k_blocks,            # k_scale: fp32 per (128 keys, head)
            4 * H * D,                   # k_mean: fp32 per (head, channel)
            8 * H * D]                   # k_sum: fp64 scratch per (head, channel)


def test_sizes_follow_the_stated_layouts(abi):
    desc = _desc(abi)
    assert abi.qk_i8_sizes(desc, H, D) == _expected_i8()
    assert abi.qk_e4m3_sizes(desc, H, D) == _expected_i8()[:4]


@pytest.mark.parametrize("sizes", ["qk_i8_sizes", "qk_e4m3_sizes"])
def test_sizes_reject_other_head_dims(abi, sizes):
    with pytest.raises(abi.WfError) as e:
        getattr(abi, sizes)(_desc(abi), H, 64)
    assert e.value.code == abi.WF_ERR_SHAPE


def _buffers(fields, sizes, short=None):
    """CPU stand-ins of the right dtypes; the field `short` one element too small."""
    dtypes = {"q_codes": torch.uint8, "k_codes": torch.uint8, "q_scale": torch.float32,
              "k_scale": torch.float32, "k_mean": torch.float32, "k_sum": torch.float64}
    out = {}
    for n, sz in zip(fields, sizes):
        dt = dtypes[n]
        count = sz // torch.empty((), dtype=dt).element_size()
        out[n] = torch.zeros(count - (1 if n == short else 0), dtype=dt)
    return out


def _call_args():
    pool = torch.zeros(8, 32, H, D, dtype=torch.bfloat16)
    return dict(q=torch.zeros(T_Q, H, D, dtype=torch.bfloat16), k_pool=pool, v_pool=pool.clone(),
                page_table_row=torch.zeros(8, dtype=torch.int32),
                out=torch.zeros(T_Q, H, D, dtype=torch.bfloat16))


def _run(abi, tier, call, qk):
    a, desc = _call_args(), _desc(abi)
    if call == "quantize":
        fn = getattr(abi, f"qk_quantize_{tier}")
        fn(a["q"], a["k_pool"], a["v_pool"], a["page_table_row"], desc, qk)
    else:
        fn = getattr(abi, f"attn_forward_{tier}")
        fn(qk, a["k_pool"], a["v_pool"], a["page_table_row"], desc, 0.088, a["out"])


@pytest.mark.parametrize("call", ["quantize", "forward"])
@pytest.mark.parametrize("tier", ["i8", "e4m3"])
def test_undersized_buffers_are_refused(abi, tier, call):
    fields = abi.QK_I8_FIELDS if tier == "i8" else abi.QK_E4M3_FIELDS
    sizes = getattr(abi, f"qk_{tier}_sizes")(_desc(abi), H, D)
    for n in fields:
        with pytest.raises(ValueError, match=f"{n}: .* needs {sizes[fields.index(n)]}"):
            _run(abi, tier, call, _buffers(fields, sizes, short=n))
    # buffers of the stated sizes pass this check and stop at the next one (CPU tensors)
    with pytest.raises(ValueError, match="expected a CUDA tensor"):
        _run(abi, tier, call, _buffers(fields, sizes))
