"""Pins for the INT8 (Sage-like) attention oracle, ``oracle/int8.py`` (CPU only).

Each pin checks the oracle against something other than itself: the quantizer against its
rounding bound, ties and saturation; the mean against a library mean; the exact integer logits
against a library matrix product of the dequantized operands; the smoothing step against the
shift invariance of exact softmax attention (the C oracle); and the whole tier against a
closed-form bound on its logit error.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import int8


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).bfloat16().float().numpy()


def test_quantizer_codes_bounds_maximum_and_rounding_error():
    rng = np.random.default_rng(0)
    x = _bf16(rng.standard_normal((300, 3, 64)) * np.exp2(rng.integers(-6, 6, (1, 3, 1))))
    codes, scale = int8.quantize_blocks(x, 128)
    assert codes.dtype == np.int8 and scale.shape == (3, 3)
    assert codes.min() >= -127 and codes.max() <= 127
    for b in range(3):
        rows = slice(128 * b, min(128 * b + 128, 300))
        for h in range(3):
            xb, cb = x[rows, h], codes[rows, h]
            a = np.abs(xb).max()
            assert scale[h, b] == np.float32(a) / np.float32(127)
            assert np.abs(cb.astype(np.int64)).max() == 127              # the maximum maps to 127
            # half a code step, plus the fp32 roundings of 127 / a, a / 127 and x * inv: each
            # relative 2^-24 of values up to 127 steps, under 2^-16 of a step together
            err = np.abs(cb * np.float64(scale[h, b]) - xb)
            assert np.all(err <= (0.5 + 2.0 ** -16) * scale[h, b] + 1e-30)


def test_ties_go_to_the_even_code_and_zero_blocks_stay_zero():
    # a block whose maximum is 127 has inv = 1 exactly, so x * inv = x
    x = np.zeros((4, 2, 8), np.float32)
    x[0, 0, :6] = [127.0, 2.5, 3.5, -2.5, -3.5, 0.5]
    codes, scale = int8.quantize_blocks(x, 128)
    assert codes[0, 0, :6].tolist() == [127, 2, 4, -2, -4, 0]
    assert scale[0, 0] == 1.0
    assert scale[1, 0] == 0 and not codes[:, 1].any()                   # head 1: all zeros
    tiny = np.full((2, 1, 4), 1e-38, np.float32)                         # 127 / a overflows
    c, s = int8.quantize_blocks(tiny, 128)
    assert s[0, 0] == 0 and not c.any()


def test_key_mean_is_the_exact_mean():
    rng = np.random.default_rng(1)
    k = _bf16(rng.standard_normal((1000, 2, 16)))
    mu = int8.key_mean(k)
    ref = k.astype(np.float64).mean(axis=0)
    assert np.all(np.abs(mu - ref) <= np.abs(ref) * 2.0 ** -23 + 1e-12)
    const = np.broadcast_to(_bf16(rng.standard_normal((1, 2, 16))), (77, 2, 16))
    assert np.array_equal(int8.key_mean(const), const[0])               # a constant is its mean


def test_integer_logits_equal_a_matrix_product_of_the_dequantized_operands():
    rng = np.random.default_rng(2)
    q = _bf16(rng.standard_normal((260, 2, 64)))
    k = _bf16(rng.standard_normal((300, 2, 64)) + 3.0)
    qc, qs, kc, ks, _ = int8.quantize_qk(q, k)
    rows = np.arange(0, 260, 7)
    for h in range(2):
        got = int8.logits_rows(qc, qs, kc, ks, rows, h, 300, 0.125)
        qd = qc[rows, h].astype(np.float64) * qs[h, rows // 128][:, None]
        kd = kc[:, h].astype(np.float64) * ks[h, np.arange(300) // 128][:, None]
        ref = 0.125 * np.matmul(qd, kd.T)
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_smoothing_leaves_exact_attention_unchanged():
    """Subtracting the key mean shifts every logit of a row by one constant: the exact (C) oracle
    gives the same attention for K and for K - mu."""
    from block_causal_streaming_b200.workloads import make_inputs, small_case
    wl = small_case("smooth", 2, 64, (40,), (50, 30), 16, seed=3)
    inp = make_inputs(wl)
    k = inp.k.float().numpy() + 2.0                                      # keys far from centred
    mu = int8.key_mean(k)
    a = oracle.attention(inp.q, k, inp.v, wl.chunk_offsets, wl.num_ctx_chunks, 0.125)
    b = oracle.attention(inp.q, int8.smooth(k, mu), inp.v, wl.chunk_offsets,
                         wl.num_ctx_chunks, 0.125)
    assert np.abs(a - b).max() <= 2e-5


def _case(seed=4):
    """A small wavefront whose keys sit far from zero (+1.5 on every channel), as projected keys
    often do: the smoothing step matters there."""
    from block_causal_streaming_b200.workloads import LayerInputs, make_inputs, small_case
    wl = small_case("int8", 2, 64, (150,), (140, 90), 16, seed=seed)
    inp = make_inputs(wl)
    k = (inp.k.float() + 1.5).bfloat16()
    return wl, LayerInputs(inp.q, k, inp.v, inp.page_table)


def test_smoothed_keys_have_zero_mean():
    wl, inp = _case()
    k = inp.k.float().numpy()
    kp = int8.smooth(k, int8.key_mean(k)).astype(np.float64)
    # each K' value carries one fp32 rounding (2^-24 relative of values ~|k|)
    assert np.abs(kp.mean(axis=0)).max() <= 4 * 2.0 ** -24 * np.abs(k).max()
    assert np.abs(k.astype(np.float64).mean(axis=0)).min() > 1.0      # the raw keys do not


def test_logit_error_is_within_the_quantization_bound():
    """|s_int8 - s| <= scale (|q|_1 dk / 2 + |k_hat|_1 dq / 2) for every (row, key), where s uses
    the smoothed keys: a closed form from the half-step rounding bound of both operands."""
    wl, inp = _case()
    q = inp.q.float().numpy()
    k = inp.k.float().numpy()
    qc, qs, kc, ks, mu = int8.quantize_qk(q, k)
    kp = int8.smooth(k, mu).astype(np.float64)
    rows = np.arange(0, wl.t_q, 5)
    n = wl.t_kv
    for h in range(wl.heads):
        got = int8.logits_rows(qc, qs, kc, ks, rows, h, n, 0.125)
        exact = 0.125 * q[rows, h].astype(np.float64) @ kp[:n, h].T
        dq = qs[h, rows // 128].astype(np.float64)[:, None]
        dk = ks[h, np.arange(n) // 128].astype(np.float64)[None, :]
        k_hat = kc[:n, h].astype(np.float64) * dk.T
        bound = 0.125 * (np.abs(q[rows, h]).sum(1)[:, None] * dk / 2
                         + np.abs(k_hat).sum(1)[None, :] * dq / 2) * (1 + 1e-6)
        assert np.all(np.abs(got - exact) <= bound)


def test_int8_attention_is_close_to_exact_attention():
    """What the INT8 tier costs in accuracy, oracle against oracle (N(0,1) values, keys shifted by
    +1.5): measured
    max-abs 0.0081, mean-abs 0.00093 on this case; the bound guards against a much worse
    encoding."""
    wl, inp = _case()
    got = int8.attention(inp.q, inp.k, inp.v, wl.chunk_offsets, wl.num_ctx_chunks, 0.125)
    ref = oracle.attention(inp.q, inp.k, inp.v, wl.chunk_offsets, wl.num_ctx_chunks, 0.125)
    err = np.abs(got - ref)
    assert err.max() <= 0.03 and err.mean() <= 0.003
    assert err.mean() > 1e-5                                              # it really quantizes


def test_selected_rows_equal_the_full_output():
    wl, inp = _case()
    full = int8.attention(inp.q, inp.k, inp.v, wl.chunk_offsets, wl.num_ctx_chunks, 0.125)
    rows = [0, 5, wl.t_q - 1, 139, 140]
    heads = [0, 1, 1, 0, 1]
    sel = int8.attention(inp.q, inp.k, inp.v, wl.chunk_offsets, wl.num_ctx_chunks, 0.125,
                         rows=rows, heads=heads)
    assert np.array_equal(sel, full[rows, heads])


def test_later_chunks_are_invisible():
    """Perturbing keys and values of later chunks leaves earlier chunks' outputs unchanged once
    the quantization is held fixed (the mask, not the quantizer, decides visibility)."""
    wl, inp = _case()
    qz = int8.quantize_qk(inp.q.float().numpy(), inp.k.float().numpy())
    base = int8.attention(inp.q, inp.k, inp.v, wl.chunk_offsets, wl.num_ctx_chunks, 0.125,
                          quantized=qz)
    off, nctx = wl.chunk_offsets, wl.num_ctx_chunks
    v2 = inp.v.float().numpy().copy()
    v2[off[nctx + 1]:] += 10.0
    kc2 = qz[2].copy()
    kc2[off[nctx + 1]:] = 127
    qz2 = (qz[0], qz[1], kc2, qz[3], qz[4])
    got = int8.attention(inp.q, inp.k, v2, off, nctx, 0.125, quantized=qz2)
    first = off[nctx + 1] - off[nctx]
    assert np.array_equal(got[:first], base[:first])
    assert not np.array_equal(got[first:], base[first:])
