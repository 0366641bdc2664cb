"""Pins for the oracle: each check ties it to something other than itself.

The rule being pinned: within a chunk attention is full; across chunks a query sees every earlier
(cleaner) chunk and never a later (noisier) one (Wave Forcing project page, "01 The design gap",
panel C; KipQuest summary of arXiv 2611.00859, "The deep dive").  Attention then reads the visible
K/V "prefix in place" (project page, "03 End-to-end KV transport", item 03 "Layout").

Pins: hand-derived golden cases, an explicit-mask-matrix brute force, the one-chunk reduction to
torch's scaled_dot_product_attention, closed forms (q = 0 gives the prefix mean and lse = ln n;
V = 1 gives 1; one-hot V exposes the softmax rows), invariants (later-chunk perturbation is
bitwise invisible, a per-head key shift changes nothing), and the paged layout's golden mapping.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16(x):
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)


def rand_case(seed, D=None, max_len=40, max_chunks=4, H=None, value_scale=1.0):
    rng = np.random.default_rng(seed)
    nc = int(rng.integers(1, max_chunks + 1))
    nctx = int(rng.integers(0, nc))
    lens = rng.integers(1, max_len + 1, size=nc).tolist()
    off = [0]
    for n in lens:
        off.append(off[-1] + n)
    H = H or int(rng.integers(1, 4))
    D = D or int(rng.choice([5, 64, 128]))
    t_kv, t_q = off[-1], off[-1] - off[nctx]
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(t_q, H, D, generator=g) * value_scale).to(torch.bfloat16)
    k = (torch.randn(t_kv, H, D, generator=g) * value_scale).to(torch.bfloat16)
    v = (torch.randn(t_kv, H, D, generator=g) * value_scale).to(torch.bfloat16)
    return q, k, v, off, nctx, 1.0 / math.sqrt(D)


def chunk_ids(off):
    ids = np.empty(off[-1], dtype=np.int64)
    for c in range(len(off) - 1):
        ids[off[c]:off[c + 1]] = c
    return ids


def brute_force(q, k, v, off, nctx, scale):
    """Dense fp64 attention over a [T_q, T_kv] boolean mask built from chunk indices."""
    qd, kd, vd = (t.to(torch.float64).numpy() for t in (q, k, v))
    ids = chunk_ids(off)
    qchunk = ids[off[nctx]:]                                 # chunk of each query token
    mask = ids[None, :] <= qchunk[:, None]                   # [T_q, T_kv]
    out = np.zeros(qd.shape)
    lse = np.zeros((qd.shape[1], qd.shape[0]))
    for h in range(qd.shape[1]):
        s = scale * qd[:, h, :] @ kd[:, h, :].T
        s = np.where(mask, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        z = e.sum(axis=1, keepdims=True)
        out[:, h, :] = (e / z) @ vd[:, h, :]
        lse[h] = (m + np.log(z))[:, 0]
    return out, lse


# --------------------------------------------------------------------------------------------
def test_hand_cases():
    cases = json.load(open(os.path.join(GOLDEN, "hand_cases.json")))["cases"]
    for c in cases:
        out, lse = oracle.attention(bf16(c["q"]), bf16(c["k"]), bf16(c["v"]), c["chunk_offsets"],
                                    c["num_ctx_chunks"], c["scale"], with_lse=True)
        np.testing.assert_allclose(out, np.asarray(c["out"]), rtol=0, atol=2e-6, err_msg=c["name"])
        np.testing.assert_allclose(lse, np.asarray(c["lse"]), rtol=0, atol=2e-6, err_msg=c["name"])


@pytest.mark.parametrize("seed", range(12))
def test_brute_force_mask_matrix(seed):
    q, k, v, off, nctx, scale = rand_case(seed)
    out, lse = oracle.attention(q, k, v, off, nctx, scale, with_lse=True)
    ref_out, ref_lse = brute_force(q, k, v, off, nctx, scale)
    np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-6)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-5)


@pytest.mark.parametrize("seed,D", [(100, 64), (101, 128), (102, 7)])
def test_single_chunk_is_full_attention(seed, D):
    """One chunk, no context: block-causal attention reduces to ordinary full attention."""
    g = torch.Generator().manual_seed(seed)
    T, H = 37, 3
    q, k, v = (torch.randn(T, H, D, generator=g).to(torch.bfloat16) for _ in range(3))
    scale = 1.0 / math.sqrt(D)
    out = oracle.attention(q, k, v, [0, T], 0, scale)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q.double().transpose(0, 1), k.double().transpose(0, 1), v.double().transpose(0, 1),
        scale=scale).transpose(0, 1).numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-6)


@pytest.mark.parametrize("seed", range(4))
def test_later_chunks_are_invisible_bitwise(seed):
    q, k, v, off, nctx, scale = rand_case(seed + 20, max_chunks=5)
    nc = len(off) - 1
    base = oracle.attention(q, k, v, off, nctx, scale)
    for i in range(nctx, nc - 1):
        k2, v2 = k.clone(), v.clone()
        sl = slice(off[i + 1], off[-1])
        k2[sl] = (torch.randn_like(k2[sl].float()) * 7).to(torch.bfloat16)
        v2[sl] = (torch.randn_like(v2[sl].float()) * 7).to(torch.bfloat16)
        got = oracle.attention(q, k2, v2, off, nctx, scale)
        rows = slice(0, off[i + 1] - off[nctx])          # query rows of chunks <= i
        assert np.array_equal(got[rows], base[rows])
        assert not np.array_equal(got[off[i + 1] - off[nctx]:], base[off[i + 1] - off[nctx]:])


def test_values_of_a_later_chunk_never_leak():
    """V nonzero only inside chunk j: every query chunk before j returns exactly 0."""
    off, nctx = [0, 9, 20, 31, 40], 1
    g = torch.Generator().manual_seed(7)
    H, D = 2, 64
    q = torch.randn(off[-1] - off[nctx], H, D, generator=g).to(torch.bfloat16)
    k = torch.randn(off[-1], H, D, generator=g).to(torch.bfloat16)
    for j in range(1, 4):
        v = torch.zeros(off[-1], H, D, dtype=torch.bfloat16)
        v[off[j]:off[j + 1]] = torch.randn(off[j + 1] - off[j], H, D, generator=g).to(torch.bfloat16)
        out = oracle.attention(q, k, v, off, nctx, 0.125)
        before = off[j] - off[nctx]
        if before > 0:
            assert np.all(out[:before] == 0.0)
        assert np.any(out[before:off[j + 1] - off[nctx]] != 0.0)


@pytest.mark.parametrize("seed", range(6))
def test_zero_queries_give_prefix_mean(seed):
    """q = 0: every visible key has weight 1/n, so out = mean of V over the visible prefix and
    lse = ln n, where n = end of the query's own chunk."""
    q, k, v, off, nctx, scale = rand_case(seed + 40)
    q = torch.zeros_like(q)
    out, lse = oracle.attention(q, k, v, off, nctx, scale, with_lse=True)
    vd = v.double().numpy()
    csum = np.concatenate([np.zeros((1,) + vd.shape[1:]), np.cumsum(vd, axis=0)])
    for c in range(nctx, len(off) - 1):
        n = off[c + 1]
        mean = csum[n] / n
        for t in range(off[c], off[c + 1]):
            r = t - off[nctx]
            np.testing.assert_allclose(out[r], mean, rtol=0, atol=1e-6)
            np.testing.assert_allclose(lse[:, r], math.log(n), rtol=0, atol=1e-6)


@pytest.mark.parametrize("seed", range(3))
def test_unit_values_give_unit_outputs(seed):
    q, k, v, off, nctx, scale = rand_case(seed + 60, value_scale=3.0)
    out = oracle.attention(q, k, torch.ones_like(v), off, nctx, scale)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-6)


@pytest.mark.parametrize("seed", range(4))
def test_softmax_rows_via_one_hot_values(seed):
    """v[j] = e_j exposes the attention probabilities: each row sums to 1, masked keys get 0,
    and visible keys are proportional to exp(scale * q.k)."""
    q, k, _, off, nctx, scale = rand_case(seed + 80, D=64, max_len=15)
    t_kv, H, D = k.shape
    assert t_kv <= D
    v = torch.zeros(t_kv, H, D, dtype=torch.bfloat16)
    for j in range(t_kv):
        v[j, :, j] = 1.0
    p = oracle.attention(q, k, v, off, nctx, scale)[:, :, :t_kv]     # [T_q, H, T_kv]
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-6)
    ids = chunk_ids(off)
    qd, kd = q.double().numpy(), k.double().numpy()
    for r in range(q.shape[0]):
        c = ids[off[nctx] + r]
        vis = ids <= c
        assert np.all(p[r][:, ~vis] == 0.0)
        for h in range(H):
            logit = scale * kd[vis, h, :] @ qd[r, h, :]
            w = np.exp(logit - logit.max())
            np.testing.assert_allclose(p[r, h, vis], w / w.sum(), rtol=0, atol=1e-6)


def test_per_head_key_shift_is_invisible():
    """Adding one vector mu_h to every key of head h adds scale*q.mu_h to a whole softmax row."""
    q, k, v, off, nctx, scale = rand_case(123, D=64, H=2)
    g = torch.Generator().manual_seed(5)
    mu = torch.randn(1, k.shape[1], k.shape[2], generator=g)
    base = oracle.attention(q, k, v, off, nctx, scale)
    shifted = oracle.attention(q, (k.float() + mu).to(torch.bfloat16), v, off, nctx, scale)
    # bf16 rounding of k + mu perturbs logits slightly; the answer itself does not move
    np.testing.assert_allclose(shifted, base, rtol=0, atol=5e-2)
    exact_mu = torch.full_like(mu, 2.0)                         # exact in bf16: no rounding
    shifted2 = oracle.attention(q, (k.float() + exact_mu).to(torch.bfloat16), v, off, nctx, scale)
    ref2, _ = brute_force(q, (k.float() + exact_mu).to(torch.bfloat16), v, off, nctx, scale)
    np.testing.assert_allclose(shifted2, ref2, rtol=0, atol=1e-6)


def test_row_selection_matches_full():
    q, k, v, off, nctx, scale = rand_case(321, D=128, H=3)
    out, lse = oracle.attention(q, k, v, off, nctx, scale, with_lse=True)
    rng = np.random.default_rng(0)
    rows = rng.integers(0, q.shape[0], size=17)
    heads = rng.integers(0, q.shape[1], size=17)
    o2, l2 = oracle.attention_rows(q, k, v, off, nctx, scale, rows, heads, with_lse=True)
    assert np.array_equal(o2, out[rows, heads])
    assert np.array_equal(l2, lse[heads, rows])


def test_rejects_malformed_descriptors():
    q, k, v, off, nctx, scale = rand_case(5)
    with pytest.raises(ValueError):
        oracle.attention(q, k, v, off, len(off) - 1, scale)           # no query chunk
    bad = list(off)
    bad[0] = 1
    with pytest.raises(ValueError):
        oracle.attention(q, k, v, bad, nctx, scale)


# ------------------------------------------------------------------------------ paged layout
def test_paging_golden_case():
    c = json.load(open(os.path.join(GOLDEN, "paging_case.json")))
    pool = np.full((c["num_pages"], c["page_size"], 1, 1), -1, dtype=np.int64)
    for start, length in c["appends"]:
        rows = np.arange(start, start + length, dtype=np.int64).reshape(length, 1, 1)
        oracle.scatter_chunk(pool, c["page_table"], start, rows)
    assert np.array_equal(pool[:, :, 0, 0], np.asarray(c["expected_pool"]))
    back = oracle.gather_logical(pool, c["page_table"], 5)
    assert np.array_equal(back[:, 0, 0], np.arange(5))


@pytest.mark.parametrize("page_size", [16, 48, 64])
def test_paging_round_trip_and_identity(page_size):
    rng = np.random.default_rng(page_size)
    H, D, lens = 2, 8, [37, 100, 5, 64]
    T = sum(lens)
    pages = (T + page_size - 1) // page_size
    data = rng.integers(0, 2 ** 16, size=(T, H, D), dtype=np.uint16)
    perm = rng.permutation(pages + 3)[:pages]
    pool = np.zeros((pages + 3, page_size, H, D), dtype=np.uint16)
    start = 0
    for n in lens:
        oracle.scatter_chunk(pool, perm, start, data[start:start + n])
        start += n
    assert np.array_equal(oracle.gather_logical(pool, perm, T), data)
    ident = np.zeros((pages, page_size, H, D), dtype=np.uint16)
    oracle.scatter_chunk(ident, np.arange(pages), 0, data)
    assert np.array_equal(ident.reshape(-1, H, D)[:T], data)
