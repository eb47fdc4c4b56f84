"""Pins for the oracle's multi-token (prefill / chunked prefill) attention.

New token i of a sequence with n cached tokens and q_len new ones sits at
position p = n - q_len + i and attends to positions lo..p (lo = 0, or
p - window + 1 with a sliding window).  The oracle is checked against:
torch's scaled_dot_product_attention in float64 with an explicit mask (a
library routine, on contiguous K/V the test builds itself); pure-Python brute
force; decode attention (itself pinned) over the context p + 1; closed forms
(identical keys give the running mean of V, a one-token window gives v_p, the
first token of a full prompt gives v_0); causality under perturbation of
later tokens; invariance under physical placement; and its error cases."""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from test_oracle_attention import brute, scatter_to_pool
from workloads import BF16, E4M3, F16, e4m3_codes, fp8_scales, normal_bits


def make_prefill(rng, lens, q_lens, hq, hkv, d, bs, fmt, spare=3):
    k_seqs = [normal_bits(rng, (n, hkv, d), fmt) for n in lens]
    v_seqs = [normal_bits(rng, (n, hkv, d), fmt) for n in lens]
    nb = sum(-(-n // bs) for n in lens) + spare
    kp, vp, tables = scatter_to_pool(k_seqs, v_seqs, bs, nb, rng, np.uint16)
    cu = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    q = normal_bits(rng, (int(cu[-1]), hq, d), fmt)
    return k_seqs, v_seqs, kp, vp, tables, cu, q


def sdpa_reference(q_rows, K, V, n, q_len, scale, window=0):
    """float64 SDPA over contiguous K/V [n][hkv][d] for q rows [q_len][hq][d]."""
    hq, hkv = q_rows.shape[1], K.shape[1]
    g = hq // hkv
    pos = np.arange(n - q_len, n)[:, None]
    t = np.arange(n)[None, :]
    allowed = t <= pos
    if window:
        allowed &= t > pos - window
    Kr = torch.from_numpy(np.repeat(K, g, axis=1)).permute(1, 0, 2)  # [hq][n][d]
    Vr = torch.from_numpy(np.repeat(V, g, axis=1)).permute(1, 0, 2)
    Q = torch.from_numpy(q_rows).permute(1, 0, 2)  # [hq][q_len][d]
    out = F.scaled_dot_product_attention(Q, Kr, Vr, attn_mask=torch.from_numpy(allowed), scale=scale)
    return out.permute(1, 0, 2).numpy()


@pytest.mark.parametrize("fmt", [F16, BF16])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2), (6, 1)])
def test_matches_sdpa_with_causal_mask(fmt, hq, hkv):
    rng = np.random.default_rng(11)
    lens = [1, 9, 16, 33, 70]
    q_lens = [1, 9, 5, 33, 20]  # full prompts and chunks on top of a cached prefix
    d, bs = 16, 16
    k_seqs, v_seqs, kp, vp, tables, cu, q = make_prefill(rng, lens, q_lens, hq, hkv, d, bs, fmt)
    scale = 0.29
    out = oracle.paged_prefill(kp, vp, fmt, q, fmt, cu, tables, np.array(lens), scale, bs)
    for s, (n, ql) in enumerate(zip(lens, q_lens)):
        want = sdpa_reference(oracle.decode(q[cu[s]:cu[s + 1]], fmt), oracle.decode(k_seqs[s], fmt),
                              oracle.decode(v_seqs[s], fmt), n, ql, scale)
        assert np.allclose(out[cu[s]:cu[s + 1]], want, rtol=0, atol=1e-12)


def test_matches_pure_python_brute_force():
    rng = np.random.default_rng(12)
    lens, q_lens = [7, 20], [3, 20]
    hq, hkv, d, bs = 2, 1, 4, 16
    k_seqs, v_seqs, kp, vp, tables, cu, q = make_prefill(rng, lens, q_lens, hq, hkv, d, bs, F16)
    out = oracle.paged_prefill(kp, vp, F16, q, F16, cu, tables, np.array(lens), 0.5, bs)
    for s, (n, ql) in enumerate(zip(lens, q_lens)):
        K, V = oracle.decode(k_seqs[s], F16), oracle.decode(v_seqs[s], F16)
        for i in range(ql):
            p = n - ql + i
            Q = oracle.decode(q[cu[s] + i], F16)
            for h in range(hq):
                want = brute(list(Q[h]), [list(K[t, 0]) for t in range(p + 1)],
                             [list(V[t, 0]) for t in range(p + 1)], 0.5)
                assert np.allclose(out[cu[s] + i, h], want, rtol=0, atol=1e-12)


def test_each_row_is_decode_over_its_prefix():
    """Row i equals decode attention with context p + 1 on the same pool."""
    rng = np.random.default_rng(13)
    lens, q_lens = [40, 17], [12, 17]
    hq, hkv, d, bs = 8, 2, 16, 16
    _, _, kp, vp, tables, cu, q = make_prefill(rng, lens, q_lens, hq, hkv, d, bs, BF16)
    out = oracle.paged_prefill(kp, vp, BF16, q, BF16, cu, tables, np.array(lens), 0.25, bs)
    for s, (n, ql) in enumerate(zip(lens, q_lens)):
        rows = np.arange(cu[s], cu[s + 1])
        ctx = np.array([n - ql + i + 1 for i in range(ql)], np.int32)
        dec = oracle.paged_decode(kp, vp, BF16, q[rows], BF16, np.repeat(tables[s:s + 1], ql, 0), ctx, 0.25, bs)
        assert np.array_equal(out[rows], dec)


@pytest.mark.parametrize("window", [0, 1, 5, 16, 100])
def test_identical_keys_give_running_mean_of_v(window):
    rng = np.random.default_rng(14)
    n, ql, hkv, hq, d, bs = 50, 30, 2, 4, 8, 16
    k = np.repeat(normal_bits(rng, (1, hkv, d), F16), n, axis=0)
    v = normal_bits(rng, (n, hkv, d), F16)
    kp, vp, tables = scatter_to_pool([k], [v], bs, 6, rng, np.uint16)
    q = normal_bits(rng, (ql, hq, d), F16)
    cu = np.array([0, ql], np.int32)
    out = oracle.paged_prefill(kp, vp, F16, q, F16, cu, tables, np.array([n]), 0.7, bs, window=window)
    V = oracle.decode(v, F16)
    for i in range(ql):
        p = n - ql + i
        lo = max(0, p - window + 1) if window else 0
        for h in range(hq):
            assert np.allclose(out[i, h], V[lo:p + 1, h // 2].mean(axis=0), rtol=0, atol=1e-12)


def test_one_token_window_and_first_prompt_token_are_exact():
    rng = np.random.default_rng(15)
    n, hq, d, bs = 23, 2, 8, 16
    k_seqs, v_seqs, kp, vp, tables, cu, q = make_prefill(rng, [n], [n], hq, 2, d, bs, BF16)
    V = oracle.decode(v_seqs[0], BF16)
    one = oracle.paged_prefill(kp, vp, BF16, q, BF16, cu, tables, np.array([n]), 1.0, bs, window=1)
    assert np.array_equal(one, V)  # attends to its own position only
    full = oracle.paged_prefill(kp, vp, BF16, q, BF16, cu, tables, np.array([n]), 1.0, bs)
    assert np.array_equal(full[0], V[0])


def test_window_at_least_context_is_no_window():
    rng = np.random.default_rng(16)
    lens, q_lens = [30, 45], [10, 45]
    _, _, kp, vp, tables, cu, q = make_prefill(rng, lens, q_lens, 4, 4, 16, 16, F16)
    a = oracle.paged_prefill(kp, vp, F16, q, F16, cu, tables, np.array(lens), 0.3, 16)
    b = oracle.paged_prefill(kp, vp, F16, q, F16, cu, tables, np.array(lens), 0.3, 16, window=45)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("window", [3, 16, 17])
def test_sliding_window_matches_sdpa_band(window):
    rng = np.random.default_rng(17)
    lens, q_lens = [40, 64], [15, 64]
    hq, hkv, d, bs = 4, 2, 16, 16
    k_seqs, v_seqs, kp, vp, tables, cu, q = make_prefill(rng, lens, q_lens, hq, hkv, d, bs, BF16)
    out = oracle.paged_prefill(kp, vp, BF16, q, BF16, cu, tables, np.array(lens), 0.2, bs, window=window)
    for s, (n, ql) in enumerate(zip(lens, q_lens)):
        want = sdpa_reference(oracle.decode(q[cu[s]:cu[s + 1]], BF16), oracle.decode(k_seqs[s], BF16),
                              oracle.decode(v_seqs[s], BF16), n, ql, 0.2, window)
        assert np.allclose(out[cu[s]:cu[s + 1]], want, rtol=0, atol=1e-12)


def test_causal_rows_ignore_later_tokens():
    """Changing K/V at positions > c changes exactly the rows with p > c."""
    rng = np.random.default_rng(18)
    n, ql, hq, d, bs = 48, 48, 2, 8, 16
    k_seqs, v_seqs, kp, vp, tables, cu, q = make_prefill(rng, [n], [ql], hq, 1, d, bs, F16)
    base = oracle.paged_prefill(kp, vp, F16, q, F16, cu, tables, np.array([n]), 0.5, bs)
    c = 29
    kp2, vp2 = kp.copy(), vp.copy()
    for t in range(c + 1, n):
        blk, off = tables[0, t // bs], t % bs
        kp2[blk, :, off, :] = normal_bits(rng, (1, d), F16)
        vp2[blk, :, off, :] = normal_bits(rng, (1, d), F16)
    new = oracle.paged_prefill(kp2, vp2, F16, q, F16, cu, tables, np.array([n]), 0.5, bs)
    assert np.array_equal(new[:c + 1], base[:c + 1])
    assert all(not np.array_equal(new[i], base[i]) for i in range(c + 1, n))


def test_physical_placement_does_not_matter():
    rng = np.random.default_rng(19)
    lens, q_lens = [33, 50], [8, 50]
    k_seqs, v_seqs, kp, vp, tables, cu, q = make_prefill(rng, lens, q_lens, 4, 2, 16, 16, BF16)
    a = oracle.paged_prefill(kp, vp, BF16, q, BF16, cu, tables, np.array(lens), 0.3, 16)
    kp2, vp2, tables2 = scatter_to_pool(k_seqs, v_seqs, 16, kp.shape[0] + 5, rng, np.uint16)
    b = oracle.paged_prefill(kp2, vp2, BF16, q, BF16, cu, tables2, np.array(lens), 0.3, 16)
    assert np.array_equal(a, b)


def test_fp8_pool_matches_sdpa_on_dequantised_values():
    rng = np.random.default_rng(20)
    lens, q_lens, hq, hkv, d, bs = [37, 20], [9, 20], 4, 2, 16, 16
    nb = 8
    kp = e4m3_codes(rng, (nb, hkv, bs, d))
    vp = e4m3_codes(rng, (nb, hkv, bs, d))
    ks, vs = fp8_scales(rng, (nb, hkv)), fp8_scales(rng, (nb, hkv))
    tables = rng.permutation(nb)[:6].reshape(2, 3).astype(np.int32)
    cu = np.array([0, 9, 29], np.int32)
    q = normal_bits(rng, (29, hq, d), BF16)
    out = oracle.paged_prefill(kp, vp, E4M3, q, BF16, cu, tables, np.array(lens), 0.25, bs,
                               k_scale=ks, v_scale=vs)
    for s, (n, ql) in enumerate(zip(lens, q_lens)):
        t = np.arange(n)
        blk, off = tables[s][t // bs], t % bs
        K = oracle.decode(kp[blk, :, off, :], E4M3) * ks[blk][:, :, None]
        V = oracle.decode(vp[blk, :, off, :], E4M3) * vs[blk][:, :, None]
        want = sdpa_reference(oracle.decode(q[cu[s]:cu[s + 1]], BF16), K, V, n, ql, 0.25)
        assert np.allclose(out[cu[s]:cu[s + 1]], want, rtol=0, atol=1e-12)


def test_empty_sequences_and_error_cases():
    rng = np.random.default_rng(21)
    lens, q_lens = [10, 16], [0, 4]
    _, _, kp, vp, tables, cu, q = make_prefill(rng, lens, q_lens, 2, 2, 8, 16, F16)
    out = oracle.paged_prefill(kp, vp, F16, q, F16, cu, tables, np.array(lens), 0.5, 16)
    assert out.shape == (4, 2, 8)
    with pytest.raises(ValueError):  # more new tokens than cached ones
        oracle.paged_prefill(kp, vp, F16, q, F16, cu, tables, np.array([10, 3]), 0.5, 16)
    bad = tables.copy()
    bad[1, 0] = kp.shape[0]
    with pytest.raises(ValueError):
        oracle.paged_prefill(kp, vp, F16, q, F16, cu, bad, np.array(lens), 0.5, 16)


def test_window_reads_no_block_before_it():
    """With a window, blocks wholly before the first row's window may be
    released (table entry -1): the result is unchanged."""
    rng = np.random.default_rng(22)
    lens, q_lens, bs = [70, 41], [1, 3], 16
    _, _, kp, vp, tables, cu, q = make_prefill(rng, lens, q_lens, 4, 2, 16, bs, BF16)
    full = oracle.paged_prefill(kp, vp, BF16, q, BF16, cu, tables, np.array(lens), 0.3, bs, window=20)
    cut = tables.copy()
    for s, (n, ql) in enumerate(zip(lens, q_lens)):
        first = max(0, n - ql - 20 + 1)
        cut[s, :first // bs] = -1
    assert (cut < 0).sum() > (tables < 0).sum()
    got = oracle.paged_prefill(kp, vp, BF16, q, BF16, cu, cut, np.array(lens), 0.3, bs, window=20)
    assert np.array_equal(full, got)
