"""Pins for the FP8 (e4m3) attention-tier oracle, ``oracle/e4m3.py`` (CPU only).

Each pin checks the oracle against something other than itself: the block quantizer against the
rounding bound of the e4m3 format, with codes decoded through PyTorch's float8_e4m3fn type;
saturation and zero blocks; the logits against a library matrix product of operands decoded the
same way; the whole tier against a closed-form bound on its logit error and against exact
attention (the C oracle)."""
import numpy as np
import torch

import oracle
from oracle import e4m3

HALF_ULP = 2.0 ** -4        # e4m3: 3 mantissa bits, half a unit in the last place, relative
SUB_HALF = 2.0 ** -10       # half the subnormal step 2^-9, in code units


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).bfloat16().float().numpy()


def _decode(codes):
    """Decode through PyTorch's own float8_e4m3fn type."""
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(
        torch.float64).numpy()


def _dequant(codes, scale, block):
    T = codes.shape[0]
    s = scale.astype(np.float64)[:, np.arange(T) // block].T[:, :, None]     # [T, H, 1]
    return _decode(codes) * s


def test_quantizer_bound_saturation_and_scales():
    rng = np.random.default_rng(0)
    x = _bf16(rng.standard_normal((300, 3, 128)) * np.exp2(rng.integers(-6, 6, (1, 3, 1))))
    codes, scale = e4m3.quantize_blocks(x, 128)
    assert codes.dtype == np.uint8 and scale.shape == (3, 3)
    deq = _dequant(codes, scale, 128)
    for b in range(3):
        rows = slice(128 * b, min(128 * b + 128, 300))
        for h in range(3):
            xb = x[rows, h].astype(np.float64)
            a = np.abs(xb).max()
            assert scale[h, b] == np.float32(a) / np.float32(448)
            assert np.abs(_decode(codes[rows, h])).max() == 448.0          # the max saturates
            err = np.abs(deq[rows, h] - xb)
            bound = (HALF_ULP * np.abs(xb) + SUB_HALF * scale[h, b]) * (1 + 2.0 ** -20)
            assert np.all(err <= bound + 1e-30)


def test_zero_and_tiny_blocks_store_zeros():
    x = np.zeros((4, 2, 8), np.float32)
    x[:, 0] = np.linspace(-3, 3, 32, dtype=np.float32).reshape(4, 8)
    codes, scale = e4m3.quantize_blocks(x, 128)
    assert scale[1, 0] == 0 and not codes[:, 1].any()                       # head 1: zeros
    tiny = np.full((2, 1, 4), 1e-38, np.float32)                             # 448 / a overflows
    c, s = e4m3.quantize_blocks(tiny, 128)
    assert s[0, 0] == 0 and not c.any()


def test_logits_equal_a_library_product_of_the_dequantized_operands():
    rng = np.random.default_rng(2)
    q = _bf16(rng.standard_normal((260, 2, 128)))
    k = _bf16(rng.standard_normal((300, 2, 128)) + 3.0)
    qc, qs, kc, ks = e4m3.quantize_qk(q, k)
    qd, kd = _dequant(qc, qs, 128), _dequant(kc, ks, 128)
    rows = np.arange(0, 260, 7)
    for h in range(2):
        got = e4m3.logits_rows(qc, qs, kc, ks, rows, h, 300, 0.125)
        ref = 0.125 * torch.from_numpy(qd[rows, h]) @ torch.from_numpy(kd[:, h]).T
        assert np.allclose(got, ref.numpy(), rtol=1e-12, atol=1e-12)


def _case(seed=4):
    from block_causal_streaming_b200.workloads import LayerInputs, make_inputs, small_case
    wl = small_case("e4m3", 2, 128, (150,), (140, 90), 16, seed=seed)
    inp = make_inputs(wl)
    return wl, LayerInputs(inp.q, (inp.k.float() + 1.5).bfloat16(), inp.v, inp.page_table)


def test_logit_error_is_within_the_quantization_bound():
    """|s_fp8 - s| <= scale sum_d (|dq_d| |k^_d| + |q_d| |dk_d|), each |d| bounded per element by
    the format's rounding bound."""
    wl, inp = _case()
    q = inp.q.float().numpy().astype(np.float64)
    k = inp.k.float().numpy().astype(np.float64)
    qc, qs, kc, ks = e4m3.quantize_qk(q.astype(np.float32), k.astype(np.float32))
    kd = _dequant(kc, ks, 128)
    rows = np.arange(0, wl.t_q, 5)
    n = wl.t_kv
    for h in range(wl.heads):
        got = e4m3.logits_rows(qc, qs, kc, ks, rows, h, n, 0.125)
        exact = 0.125 * q[rows, h] @ k[:n, h].T
        dq = HALF_ULP * np.abs(q[rows, h]) + SUB_HALF * qs[h, rows // 128][:, None]
        dk = HALF_ULP * np.abs(k[:n, h]) + SUB_HALF * ks[h, np.arange(n) // 128][:, None]
        bound = 0.125 * (dq @ np.abs(kd[:n, h]).T + np.abs(q[rows, h]) @ dk.T) * (1 + 1e-6)
        assert np.all(np.abs(got - exact) <= bound)


def test_fp8_attention_is_close_to_exact_attention():
    """What the tier costs in accuracy, oracle against oracle (N(0,1) values, keys shifted by
    +1.5): measured max-abs 0.111, mean-abs 0.0077 on this case -- about 8 x the INT8 tier's,
    since e4m3 keeps 3 mantissa bits per value; the bound guards against a much worse encoding."""
    wl, inp = _case()
    got = e4m3.attention(inp.q, inp.k, inp.v, wl.chunk_offsets, wl.num_ctx_chunks, 0.125)
    ref = oracle.attention(inp.q, inp.k, inp.v, wl.chunk_offsets, wl.num_ctx_chunks, 0.125)
    err = np.abs(got - ref)
    assert err.max() <= 0.25 and err.mean() <= 0.02
    assert err.mean() > 1e-5                                              # it really quantizes


def test_selected_rows_equal_the_full_output():
    wl, inp = _case()
    full = e4m3.attention(inp.q, inp.k, inp.v, wl.chunk_offsets, wl.num_ctx_chunks, 0.125)
    rows = [0, 5, wl.t_q - 1, 139, 140]
    heads = [0, 1, 1, 0, 1]
    sel = e4m3.attention(inp.q, inp.k, inp.v, wl.chunk_offsets, wl.num_ctx_chunks, 0.125,
                         rows=rows, heads=heads)
    assert np.array_equal(sel, full[rows, heads])


def test_later_chunks_are_invisible():
    wl, inp = _case()
    qz = e4m3.quantize_qk(inp.q.float().numpy(), inp.k.float().numpy())
    base = e4m3.attention(inp.q, inp.k, inp.v, wl.chunk_offsets, wl.num_ctx_chunks, 0.125,
                          quantized=qz)
    off, nctx = wl.chunk_offsets, wl.num_ctx_chunks
    v2 = inp.v.float().numpy().copy()
    v2[off[nctx + 1]:] += 10.0
    kc2 = qz[2].copy()
    kc2[off[nctx + 1]:] = 0x7E
    got = e4m3.attention(inp.q, inp.k, v2, off, nctx, 0.125, quantized=(qz[0], qz[1], kc2, qz[3]))
    first = off[nctx + 1] - off[nctx]
    assert np.array_equal(got[:first], base[:first])
    assert not np.array_equal(got[first:], base[first:])
