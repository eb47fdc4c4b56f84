"""Pins for the oracle's paged decode attention.

The oracle rebuilds each sequence's contiguous K/V from the block table and
runs textbook softmax attention.  It is checked against: pure-Python brute
force on contiguous lists; torch's scaled_dot_product_attention in float64
(a library routine); closed forms (one token, identical keys, zero query);
invariance under physical placement and under sharing vs copying blocks; the
split-K merge identity; and GQA expressed as MHA on repeated KV heads."""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from workloads import BF16, E4M3, F16, e4m3_codes, fp8_scales, normal_bits


def scatter_to_pool(k_seqs, v_seqs, bs, num_blocks, rng, fmt_dtype):
    """Test-side inverse of paging: write each sequence's contiguous rows into
    a pool at randomly chosen physical blocks; returns pools and tables."""
    hkv, d = k_seqs[0].shape[1], k_seqs[0].shape[2]
    kp = np.zeros((num_blocks, hkv, bs, d), dtype=fmt_dtype)
    vp = np.zeros_like(kp)
    need = [-(-k.shape[0] // bs) for k in k_seqs]
    perm = rng.permutation(num_blocks)
    width = max(max(need), 1)
    tables = np.full((len(k_seqs), width), -1, dtype=np.int32)
    off = 0
    for s, (k, v) in enumerate(zip(k_seqs, v_seqs)):
        for i in range(need[s]):
            blk = perm[off]
            off += 1
            tables[s, i] = blk
            rows = slice(i * bs, min((i + 1) * bs, k.shape[0]))
            n = rows.stop - rows.start
            kp[blk, :, :n, :] = np.transpose(k[rows], (1, 0, 2))
            vp[blk, :, :n, :] = np.transpose(v[rows], (1, 0, 2))
    return kp, vp, tables


def make_case(rng, lens, hq, hkv, d, bs, fmt, spare=3):
    k_seqs = [normal_bits(rng, (n, hkv, d), fmt) for n in lens]
    v_seqs = [normal_bits(rng, (n, hkv, d), fmt) for n in lens]
    nb = sum(-(-n // bs) for n in lens) + spare
    kp, vp, tables = scatter_to_pool(k_seqs, v_seqs, bs, nb, rng, np.uint16)
    q = normal_bits(rng, (len(lens), hq, d), fmt)
    return k_seqs, v_seqs, kp, vp, tables, q


def brute(qrow, krows, vrows, scale):
    z = [scale * sum(a * b for a, b in zip(qrow, k)) for k in krows]
    m = max(z)
    w = [math.exp(x - m) for x in z]
    tot = sum(w)
    return [sum(w[t] * vrows[t][j] for t in range(len(w))) / tot for j in range(len(qrow))]


@pytest.mark.parametrize("fmt", [F16, BF16])
def test_matches_pure_python_brute_force(fmt):
    rng = np.random.default_rng(1)
    lens = [1, 5, 16, 17, 40]
    hq, hkv, d, bs = 4, 2, 8, 16
    k_seqs, v_seqs, kp, vp, tables, q = make_case(rng, lens, hq, hkv, d, bs, fmt)
    scale = 0.37
    out = oracle.paged_decode(kp, vp, fmt, q, fmt, tables, np.array(lens), scale, bs)
    g = hq // hkv
    for s, n in enumerate(lens):
        K = oracle.decode(k_seqs[s], fmt)
        V = oracle.decode(v_seqs[s], fmt)
        Q = oracle.decode(q[s], fmt)
        for h in range(hq):
            want = brute(list(Q[h]), [list(K[t, h // g]) for t in range(n)],
                         [list(V[t, h // g]) for t in range(n)], scale)
            assert np.allclose(out[s, h], want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2), (8, 1)])
def test_matches_torch_sdpa_float64(hq, hkv):
    rng = np.random.default_rng(2 + hq + hkv)
    lens = [3, 31, 64, 129, 77]
    d, bs = 32, 16
    k_seqs, v_seqs, kp, vp, tables, q = make_case(rng, lens, hq, hkv, d, bs, BF16)
    scale = 1 / math.sqrt(d)
    out = oracle.paged_decode(kp, vp, BF16, q, BF16, tables, np.array(lens), scale, bs)
    g = hq // hkv
    for s, n in enumerate(lens):
        K = torch.from_numpy(oracle.decode(k_seqs[s], BF16)).permute(1, 0, 2)  # [hkv][n][d]
        V = torch.from_numpy(oracle.decode(v_seqs[s], BF16)).permute(1, 0, 2)
        K = K.repeat_interleave(g, dim=0)
        V = V.repeat_interleave(g, dim=0)
        Q = torch.from_numpy(oracle.decode(q[s], BF16)).unsqueeze(1)  # [hq][1][d]
        ref = F.scaled_dot_product_attention(Q, K, V, scale=scale).squeeze(1).numpy()
        assert np.allclose(out[s], ref, rtol=0, atol=1e-12)


def test_single_token_returns_that_value_row():
    rng = np.random.default_rng(3)
    k_seqs, v_seqs, kp, vp, tables, q = make_case(rng, [1, 1], 2, 2, 16, 16, F16)
    out = oracle.paged_decode(kp, vp, F16, q, F16, tables, np.array([1, 1]), 0.25, 16)
    for s in range(2):
        assert np.array_equal(out[s], oracle.decode(v_seqs[s][0], F16))


def test_identical_keys_and_zero_query_give_the_mean():
    rng = np.random.default_rng(4)
    n, d, bs = 37, 16, 16
    k = np.repeat(normal_bits(rng, (1, 1, d), F16), n, axis=0)
    v = normal_bits(rng, (n, 1, d), F16)
    kp, vp, tables = scatter_to_pool([k], [v], bs, 8, rng, np.uint16)
    q = normal_bits(rng, (1, 1, d), F16)
    out = oracle.paged_decode(kp, vp, F16, q, F16, tables, np.array([n]), 0.5, bs)
    mean = oracle.decode(v, F16)[:, 0, :].mean(axis=0)
    assert np.allclose(out[0, 0], mean, rtol=0, atol=1e-12)
    # a zero query makes every logit zero: again the plain mean of V
    k2 = normal_bits(rng, (n, 1, d), F16)
    kp2, vp2, tables2 = scatter_to_pool([k2], [v], bs, 8, rng, np.uint16)
    out2 = oracle.paged_decode(kp2, vp2, F16, np.zeros((1, 1, d), np.uint16), F16, tables2,
                               np.array([n]), 0.5, bs)
    assert np.allclose(out2[0, 0], mean, rtol=0, atol=1e-12)


def test_physical_placement_does_not_change_the_output():
    rng = np.random.default_rng(5)
    lens = [50, 3, 100]
    k_seqs = [normal_bits(rng, (n, 2, 16), BF16) for n in lens]
    v_seqs = [normal_bits(rng, (n, 2, 16), BF16) for n in lens]
    q = normal_bits(rng, (3, 2, 16), BF16)
    outs = []
    for seed in (10, 11, 12):
        kp, vp, tables = scatter_to_pool(k_seqs, v_seqs, 16, 20, np.random.default_rng(seed), np.uint16)
        outs.append(oracle.paged_decode(kp, vp, BF16, q, BF16, tables, np.array(lens), 0.3, 16))
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])


def test_shared_blocks_equal_private_copies():
    rng = np.random.default_rng(6)
    bs, d = 16, 16
    nb = 12
    kp = normal_bits(rng, (nb, 1, bs, d), F16)
    vp = normal_bits(rng, (nb, 1, bs, d), F16)
    # two sequences share physical blocks 0,1 (prefix), then diverge
    shared = np.array([[0, 1, 2, -1], [0, 1, 3, -1]], dtype=np.int32)
    # the same logical content with the prefix copied into private blocks
    kp2, vp2 = kp.copy(), vp.copy()
    for src, dst in ((0, 4), (1, 5)):
        kp2[dst], vp2[dst] = kp[src], vp[src]
    private = np.array([[0, 1, 2, -1], [4, 5, 3, -1]], dtype=np.int32)
    q = normal_bits(rng, (2, 1, d), F16)
    lens = np.array([40, 45])
    a = oracle.paged_decode(kp, vp, F16, q, F16, shared, lens, 0.25, bs)
    b = oracle.paged_decode(kp2, vp2, F16, q, F16, private, lens, 0.25, bs)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("part", [16, 48, 512])
def test_split_partials_merge_to_the_unsplit_result(part):
    rng = np.random.default_rng(7)
    lens = [1, 16, 47, 600, 1025, 0]
    k_seqs, v_seqs, kp, vp, tables, q = make_case(rng, [max(n, 1) for n in lens], 4, 2, 32, 16, BF16)
    cl = np.array(lens)
    full = oracle.paged_decode(kp, vp, BF16, q, BF16, tables, cl, 0.2, 16)
    nparts = -(-max(lens) // part)
    o, m, l = oracle.paged_decode_partials(kp, vp, BF16, q, BF16, tables, cl, 0.2, 16, part, nparts)
    merged = oracle.lse_merge(o, m, l)
    assert np.allclose(merged, full, rtol=0, atol=1e-12)
    assert np.all(merged[5] == 0)  # empty context -> zeros
    # partitions past the end are empty
    assert np.all(np.isneginf(m[0, :, 1:])) and np.all(l[0, :, 1:] == 0)


def test_fp8_pool_is_the_dequantised_pool():
    rng = np.random.default_rng(8)
    nb, hkv, bs, d = 10, 2, 16, 32
    kp = e4m3_codes(rng, (nb, hkv, bs, d))
    vp = e4m3_codes(rng, (nb, hkv, bs, d))
    ks = fp8_scales(rng, (nb, hkv))
    vs = fp8_scales(rng, (nb, hkv))
    tables = rng.permutation(nb).astype(np.int32)[:8].reshape(2, 4)
    lens = np.array([60, 33])
    q = normal_bits(rng, (2, 4, d), BF16)
    out = oracle.paged_decode(kp, vp, E4M3, q, BF16, tables, lens, 0.1, bs, ks, vs)
    # reference: dequantise with torch's float8 decode, then SDPA in float64
    K = torch.from_numpy(kp).view(torch.float8_e4m3fn).double() * torch.from_numpy(ks).double()[:, :, None, None]
    V = torch.from_numpy(vp).view(torch.float8_e4m3fn).double() * torch.from_numpy(vs).double()[:, :, None, None]
    for s in range(2):
        n = lens[s]
        blk = torch.from_numpy(tables[s])
        Ks = K[blk].permute(1, 0, 2, 3).reshape(hkv, -1, d)[:, :n].repeat_interleave(2, dim=0)
        Vs = V[blk].permute(1, 0, 2, 3).reshape(hkv, -1, d)[:, :n].repeat_interleave(2, dim=0)
        Q = torch.from_numpy(oracle.decode(q[s], BF16)).unsqueeze(1)
        ref = F.scaled_dot_product_attention(Q, Ks, Vs, scale=0.1).squeeze(1).numpy()
        assert np.allclose(out[s], ref, rtol=0, atol=1e-12)


def test_zero_context_gives_zeros_and_bad_block_is_an_error():
    rng = np.random.default_rng(9)
    k_seqs, v_seqs, kp, vp, tables, q = make_case(rng, [20, 20], 2, 2, 16, 16, F16)
    out = oracle.paged_decode(kp, vp, F16, q, F16, tables, np.array([0, 20]), 0.25, 16)
    assert np.all(out[0] == 0)
    bad = tables.copy()
    bad[1, 1] = kp.shape[0] + 5
    with pytest.raises(ValueError):
        oracle.paged_decode(kp, vp, F16, q, F16, bad, np.array([0, 20]), 0.25, 16)
