"""The FP8 (e4m3) attention tier on the GPU against its oracle (``oracle/e4m3.py``).

The quantization decides codes, so the e4m3 codes and the fp32 scales must equal the oracle's
bit for bit; the attention over the codes (QK^T on tcgen05 kind::f8f6f4 with fp32 accumulation)
must meet the parity bar (max-abs 1e-2, mean-abs 1e-3) against the oracle's FP8-tier attention.
Small cases are compared on every element, the 1.3B 5-step wavefront on whole units and sampled
rows.
"""
import numpy as np
import pytest
import torch

from oracle import e4m3 as oe4
from block_causal_streaming_b200 import WF_ERR_SHAPE, WF_OK, WfError, check_status
from block_causal_streaming_b200.layer import QkE4m3Buffers
from block_causal_streaming_b200.workloads import (WAN13B_5STEP, LayerInputs, make_inputs,
                                                   small_case)
from gpu_util import assert_parity, place, sample_rows, scale_of, whole_units

pytestmark = pytest.mark.gpu

CASES = [
    small_case("e4m3_ctx2_act3", 2, 128, (300, 200), (257, 300, 129), 64, seed=181),
    small_case("e4m3_tq_below_tile", 3, 128, (500,), (20,), 128, seed=182),
    small_case("e4m3_short_chunks_ps16", 2, 128, (37,), (5, 1, 130, 70), 16, seed=183),
    small_case("e4m3_empty_chunk", 1, 128, (90,), (100, 0, 250), 32, seed=184),
]


def _shifted(inp, shift=1.5):
    return LayerInputs(inp.q, (inp.k.float() + shift).bfloat16(), inp.v, inp.page_table)


def _run(wl, inp, fill=None):
    layer, q, _, _ = place(wl, inp, fill=fill)
    qk = QkE4m3Buffers(layer.desc, wl.heads, wl.head_dim, "cuda")
    out = torch.empty_like(q)
    layer.forward_e4m3(q, out, qk, scale=scale_of(wl))
    return layer, q, qk, out


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_quantization_is_bit_exact(wl):
    inp = _shifted(make_inputs(wl))
    _, _, qk, _ = _run(wl, inp, fill=float("nan"))
    assert check_status() == WF_OK
    qc, qs, kc, ks = oe4.quantize_qk(inp.q.float().numpy(), inp.k.float().numpy())
    assert np.array_equal(qk.k_codes.cpu().numpy(), kc)
    assert np.array_equal(qk.k_scale.cpu().numpy().view(np.int32), ks.reshape(-1).view(np.int32))
    assert np.array_equal(qk.q_codes.cpu().numpy(), qc)
    assert np.array_equal(qk.q_scale.cpu().numpy().view(np.int32), qs.reshape(-1).view(np.int32))


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_fp8_attention_every_element(wl):
    inp = _shifted(make_inputs(wl))
    _, _, _, out = _run(wl, inp, fill=float("nan"))
    assert check_status() == WF_OK
    ref = oe4.attention(inp.q, inp.k, inp.v, wl.chunk_offsets, wl.num_ctx_chunks, scale_of(wl))
    assert_parity(out.float().cpu().numpy(), ref, wl.name)


def test_later_chunks_are_invisible_and_runs_repeat_bitwise():
    from block_causal_streaming_b200 import attn_forward_e4m3
    wl = CASES[0]
    inp = _shifted(make_inputs(wl))
    layer, q, qk, out = _run(wl, inp)
    out2 = torch.empty_like(out)
    attn_forward_e4m3(qk, layer.pool.k, layer.pool.v, layer.page_tables[0], layer.desc,
                      scale_of(wl), out2)
    assert torch.equal(out, out2)
    off, nctx = wl.chunk_offsets, wl.num_ctx_chunks
    v2 = inp.v.clone()
    v2[off[nctx + 1]:] = (v2[off[nctx + 1]:].float() * 7 + 3).bfloat16()
    layer.append_range(inp.k.cuda(), v2.cuda(), range(nctx + 1, wl.num_chunks))
    out3 = torch.empty_like(out)
    attn_forward_e4m3(qk, layer.pool.k, layer.pool.v, layer.page_tables[0], layer.desc,
                      scale_of(wl), out3)
    first = off[nctx + 1] - off[nctx]
    assert check_status() == WF_OK
    assert torch.equal(out3[:first], out[:first])
    assert not torch.equal(out3[first:], out[first:])


def test_full_size_wavefront_fp8_parity():
    """The 1.3B 5-step wavefront: quantization bit-exact, attention on two whole units (every
    head) and sampled rows."""
    wl = WAN13B_5STEP
    inp = _shifted(make_inputs(wl), 0.75)
    _, _, qk, out = _run(wl, inp)
    assert check_status() == WF_OK
    quant = oe4.quantize_qk(inp.q.float().numpy(), inp.k.float().numpy())
    assert np.array_equal(qk.k_codes.cpu().numpy(), quant[2])
    assert np.array_equal(qk.q_codes.cpu().numpy(), quant[0])
    u_rows, u_heads, units = whole_units(wl, seed=7, interior=False)
    keep = np.isin(u_rows // 256, units[-2:])
    s_rows, s_heads = sample_rows(wl, per_chunk=3, seed=7)
    rows = np.concatenate([u_rows[keep], np.asarray(s_rows, np.int32)])
    heads = np.concatenate([u_heads[keep], np.asarray(s_heads, np.int32)])
    ref = oe4.attention(inp.q, inp.k, inp.v, wl.chunk_offsets, wl.num_ctx_chunks, scale_of(wl),
                        rows=rows, heads=heads, quantized=quant)
    mx, mean = assert_parity(out[rows, heads].float().cpu().numpy(), ref, wl.name)
    print(f"FP8 tier, {wl.name}: {len(rows)} (row, head) pairs: max-abs {mx:.3e}, "
          f"mean-abs {mean:.3e}")


def test_head_dim_64_is_rejected():
    wl = small_case("e4m3_d64", 2, 64, (40,), (30,), 16, seed=185)
    layer, q, _, _ = place(wl, make_inputs(wl))
    with pytest.raises(WfError) as e:
        QkE4m3Buffers(layer.desc, wl.heads, wl.head_dim, "cuda")
    assert e.value.code == WF_ERR_SHAPE
