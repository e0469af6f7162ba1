"""Pins for the fp64 CPU oracle (no GPU).

Each test checks the oracle against something other than itself: a closed
form, an invariant the mathematics fixes, a library routine on a special
case, brute force on tiny inputs, or numbers printed on the pages.  Both
oracle implementations (numpy and the threaded C file) are checked.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import attention as npo
from oracle import c_oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
IMPLS = ["numpy", "c"]


def run(impl, q, k, v, skv, scale, causal):
    if impl == "numpy":
        return npo.attention_fwd(q, k, v, skv, scale, causal)
    return c_oracle.attention_fwd(q, k, v, skv, scale, causal, nthreads=4)


def rnd(shape, seed, scale=1.0):
    g = np.random.default_rng(seed)
    # float32-representable values so both oracles see identical inputs
    return (g.standard_normal(shape) * scale).astype(np.float32).astype(np.float64)


# ---------------------------------------------------------------- library pins

@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (6, 1)])
def test_matches_torch_sdpa_fp64(impl, causal, Hq, Hkv):
    """Sq == Skv: torch's SDPA (fp64, CPU, enable_gqa) is an independent
    library routine for exactly this function ("zdabc.icu" MQA article,
    bench_mqa.py's native path)."""
    B, S, d, dv = 2, 37, 16, 12
    q, k, v = rnd((B, Hq, S, d), 1), rnd((B, Hkv, S, d), 2), rnd((B, Hkv, S, dv), 3)
    scale = 1 / math.sqrt(d)
    out, lse = run(impl, q, k, v, [S] * B, scale, causal)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
        is_causal=causal, scale=scale, enable_gqa=True).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)
    # LSE against torch.logsumexp of library-computed scores
    kr = torch.from_numpy(k).repeat_interleave(Hq // Hkv, dim=1)
    s = scale * torch.from_numpy(q) @ kr.transpose(-1, -2)
    if causal:
        s = s.masked_fill(torch.ones(S, S, dtype=torch.bool).triu(1), -math.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("impl", IMPLS)
def test_decode_varlen_matches_sdpa_per_sequence(impl):
    """Sq = 1 (decode) with ragged lengths: bottom-right causal alignment
    means the single query sees every key, so each sequence equals SDPA
    without a mask over its own first skv_b rows."""
    B, Hq, Hkv, S, d, dv = 3, 8, 2, 29, 16, 16
    q, k, v = rnd((B, Hq, 1, d), 4), rnd((B, Hkv, S, d), 5), rnd((B, Hkv, S, dv), 6)
    skv = [29, 1, 17]
    out, lse = run(impl, q, k, v, skv, 0.3, True)
    for b, L in enumerate(skv):
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[b:b + 1]), torch.from_numpy(k[b:b + 1, :, :L]),
            torch.from_numpy(v[b:b + 1, :, :L]), scale=0.3, enable_gqa=True).numpy()
        np.testing.assert_allclose(out[b:b + 1], ref, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------- head-sharing pins

@pytest.mark.parametrize("impl", IMPLS)
def test_gqa_equals_mha_on_repeated_kv(impl):
    """MQA/GQA equals MHA over K/V materialised with repeat_interleave
    ("GQA和MLA详解" section 2; "Full 路线" section 三 repeat_kv): bitwise in
    fp64, since the arithmetic is the same."""
    B, Hq, Hkv, S, d = 2, 8, 2, 19, 8
    q, k, v = rnd((B, Hq, 5, d), 7), rnd((B, Hkv, S, d), 8), rnd((B, Hkv, S, d), 9)
    skv = [19, 11]
    o1, l1 = run(impl, q, k, v, skv, 0.5, True)
    o2, l2 = run(impl, q, npo.repeat_kv(k, 4), npo.repeat_kv(v, 4), skv, 0.5, True)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
    # the other plausible mapping (head h -> kv head h % Hkv) is a different
    # function: the pin above would catch it
    o3, _ = run(impl, q, np.tile(k, (1, 4, 1, 1)), np.tile(v, (1, 4, 1, 1)), skv, 0.5, True)
    assert not np.allclose(o1, o3)


# ----------------------------------------------------------- softmax pins

def test_softmax_rows_sum_to_one():
    """Weights are a probability distribution over the visible keys
    ("带你了解Attention" section 1.2)."""
    q, k = rnd((2, 4, 9, 8), 10, 3.0), rnd((2, 2, 13, 8), 11, 3.0)
    for b, P in enumerate(npo.softmax_probs(q, k, [13, 9], 0.7, True)):
        sums = P.sum(-1)
        np.testing.assert_allclose(sums, 1.0, atol=1e-15 * 16)
        assert (P >= 0).all()


@pytest.mark.parametrize("impl", IMPLS)
def test_constant_v_gives_that_row(impl):
    q, k = rnd((2, 4, 7, 8), 12, 2.0), rnd((2, 1, 11, 8), 13, 2.0)
    row = rnd((6,), 14)
    v = np.broadcast_to(row, (2, 1, 11, 6)).copy()
    out, _ = run(impl, q, k, v, [11, 7], 0.4, True)  # every causal row sees >= 1 key
    np.testing.assert_allclose(out, np.broadcast_to(row, out.shape), rtol=0, atol=1e-14)


@pytest.mark.parametrize("impl", IMPLS)
def test_identity_v_returns_weights(impl):
    """v_j = e_j (Skv = d_v) makes the output row the weight row itself."""
    S = 10
    q, k = rnd((1, 2, 4, 8), 15), rnd((1, 1, S, 8), 16)
    v = np.eye(S)[None, None]
    out, _ = run(impl, q, k, v, [S], 0.9, False)
    P = npo.softmax_probs(q, k, [S], 0.9, False)[0]
    np.testing.assert_allclose(out[0], P, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("impl", IMPLS)
def test_first_causal_row_is_v0(impl):
    """Causal row 0 (Sq == Skv) sees only key 0: out = v_0, lse = scale q0.k0
    ("GQA和MLA详解" section 1, causal mask)."""
    q, k, v = rnd((1, 3, 6, 8), 17), rnd((1, 3, 6, 8), 18), rnd((1, 3, 6, 5), 19)
    out, lse = run(impl, q, k, v, [6], 0.25, True)
    np.testing.assert_array_equal(out[0, :, 0], v[0, :, 0])
    np.testing.assert_allclose(lse[0, :, 0], 0.25 * np.einsum("hd,hd->h", q[0, :, 0], k[0, :, 0]),
                               rtol=1e-15, atol=1e-15)


@pytest.mark.parametrize("impl", IMPLS)
def test_zero_query_uniform_weights(impl):
    """Q = 0: every visible key has weight 1/n, so out = mean of visible V
    rows and lse = ln n (causal row i with Sq = Skv: n = i + 1)."""
    S = 9
    q = np.zeros((1, 2, S, 8))
    k, v = rnd((1, 1, S, 8), 20), rnd((1, 1, S, 4), 21)
    out, lse = run(impl, q, k, v, [S], 1.0, True)
    for i in range(S):
        np.testing.assert_allclose(out[0, :, i], np.broadcast_to(v[0, 0, :i + 1].mean(0), (2, 4)),
                                   rtol=1e-14, atol=1e-15)
        np.testing.assert_allclose(lse[0, :, i], math.log(i + 1), rtol=0, atol=1e-14)


@pytest.mark.parametrize("impl", IMPLS)
def test_skv_one_and_empty(impl):
    q, k, v = rnd((2, 2, 1, 8), 22), rnd((2, 1, 3, 8), 23), rnd((2, 1, 3, 4), 24)
    out, lse = run(impl, q, k, v, [1, 0], 0.5, True)
    np.testing.assert_array_equal(out[0, :, 0], np.broadcast_to(v[0, 0, 0], (2, 4)))
    np.testing.assert_allclose(lse[0, :, 0], 0.5 * q[0, :, 0] @ k[0, 0, 0], rtol=1e-15)
    assert (out[1] == 0).all() and np.isneginf(lse[1]).all()


# ------------------------------------------------------------ invariances

@pytest.mark.parametrize("impl", IMPLS)
def test_key_shift(impl):
    """Adding w to every key adds scale*q.w to each score of a row: the
    weights are unchanged and lse moves by exactly scale*q.w."""
    q, k, v = rnd((1, 4, 5, 8), 25), rnd((1, 2, 12, 8), 26), rnd((1, 2, 12, 6), 27)
    w = rnd((8,), 28)
    # dyadic values so k + w is exact in the C oracle's float32 inputs too
    k, w = np.round(k * 64) / 64, np.round(w * 64) / 64
    o1, l1 = run(impl, q, k, v, [12], 0.6, True)
    o2, l2 = run(impl, q, k + w, v, [12], 0.6, True)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l2 - l1, 0.6 * np.einsum("bhid,d->bhi", q, w), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("impl", IMPLS)
def test_key_permutation_noncausal(impl):
    q, k, v = rnd((1, 4, 3, 8), 29), rnd((1, 1, 15, 8), 30), rnd((1, 1, 15, 6), 31)
    perm = np.random.default_rng(0).permutation(15)
    o1, l1 = run(impl, q, k, v, [15], 0.5, False)
    o2, l2 = run(impl, q, k[:, :, perm], v[:, :, perm], [15], 0.5, False)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(l2, l1, rtol=1e-13, atol=1e-14)


def test_split_combine_equals_unsplit():
    """Any partition of the keys, merged with the LSE-weighted combine, gives
    the unsplit result (the algebra the split-KV decode relies on)."""
    q, k, v = rnd((1, 4, 1, 16), 32, 2.0), rnd((1, 1, 50, 16), 33, 2.0), rnd((1, 1, 50, 8), 34)
    full_o, full_l = npo.attention_fwd(q, k, v, [50], 0.5, False)
    for bounds in ([0, 50], [0, 7, 50], [0, 1, 2, 30, 49, 50], [0, 25, 25, 50]):
        parts_o, parts_l = [], []
        for a, b in zip(bounds[:-1], bounds[1:]):
            o, l = npo.attention_fwd(q, k[:, :, a:b], v[:, :, a:b], [b - a], 0.5, False)
            parts_o.append(o)
            parts_l.append(l)
        o, l = npo.split_combine(np.stack(parts_o), np.stack(parts_l))
        np.testing.assert_allclose(o, full_o, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(l, full_l, rtol=1e-13, atol=1e-14)
    o, l = npo.split_combine(np.zeros((2, 3, 4)), np.full((2, 3), -np.inf))
    assert (o == 0).all() and np.isneginf(l).all()


# ------------------------------------------------------------- brute force

@pytest.mark.parametrize("impl", IMPLS)
def test_two_keys_closed_form(impl):
    """Skv = 2: out = (e^a v0 + e^b v1) / (e^a + e^b), lse = ln(e^a + e^b)."""
    q, k, v = rnd((1, 1, 1, 3), 35), rnd((1, 1, 2, 3), 36), rnd((1, 1, 2, 4), 37)
    out, lse = run(impl, q, k, v, [2], 0.8, False)
    a = 0.8 * sum(q[0, 0, 0, t] * k[0, 0, 0, t] for t in range(3))
    b = 0.8 * sum(q[0, 0, 0, t] * k[0, 0, 1, t] for t in range(3))
    ea, eb = math.exp(a), math.exp(b)
    for c in range(4):
        assert abs(out[0, 0, 0, c] - (ea * v[0, 0, 0, c] + eb * v[0, 0, 1, c]) / (ea + eb)) < 1e-14
    assert abs(lse[0, 0, 0] - math.log(ea + eb)) < 1e-14


@pytest.mark.parametrize("impl", IMPLS)
def test_brute_force_tiny_causal_gqa(impl):
    """Enumerate every (b, h, i, j) on a tiny ragged causal GQA case with
    plain loops and math.exp."""
    B, Hq, Hkv, Sq, d, dv = 2, 4, 2, 3, 2, 2
    skv = [3, 5]
    q, k, v = rnd((B, Hq, Sq, d), 38), rnd((B, Hkv, 5, d), 39), rnd((B, Hkv, 5, dv), 40)
    out, lse = run(impl, q, k, v, skv, 0.9, True)
    for b in range(B):
        for h in range(Hq):
            kv = h // (Hq // Hkv)
            for i in range(Sq):
                js = [j for j in range(skv[b]) if j <= i + skv[b] - Sq]
                w = [math.exp(0.9 * sum(q[b, h, i, t] * k[b, kv, j, t] for t in range(d))) for j in js]
                Z = sum(w)
                for c in range(dv):
                    ref = sum(wj * v[b, kv, j, c] for wj, j in zip(w, js)) / Z
                    assert abs(out[b, h, i, c] - ref) < 1e-13
                assert abs(lse[b, h, i] - math.log(Z)) < 1e-13


@pytest.mark.parametrize("impl", IMPLS)
def test_extend_equals_token_by_token_decode(impl):
    """Bottom-right alignment is what makes a chunk of Sq new tokens against
    a cache the same as decoding them one at a time: query i of the chunk
    equals a single decode query against the first skv - Sq + i + 1 keys
    (decode itself is pinned to SDPA above).  Includes skv < Sq, where the
    first queries see no key at all."""
    B, Hq, Hkv, Sq, d, dv = 3, 4, 2, 4, 8, 6
    q, k, v = rnd((B, Hq, Sq, d), 41), rnd((B, Hkv, 12, d), 42), rnd((B, Hkv, 12, dv), 43)
    skv = [12, 4, 2]
    out, lse = run(impl, q, k, v, skv, 0.6, True)
    for b, L in enumerate(skv):
        for i in range(Sq):
            n = L - Sq + i + 1  # keys in the cache when token i arrives
            if n <= 0:
                assert (out[b, :, i] == 0).all() and np.isneginf(lse[b, :, i]).all()
                continue
            o1, l1 = run(impl, q[b:b + 1, :, i:i + 1], k[b:b + 1, :, :n], v[b:b + 1, :, :n],
                         [n], 0.6, True)
            np.testing.assert_allclose(out[b, :, i], o1[0, :, 0], rtol=1e-13, atol=1e-14)
            np.testing.assert_allclose(lse[b, :, i], l1[0, :, 0], rtol=1e-13, atol=1e-14)


# ----------------------------------------------------------------- MLA

def test_mla_absorption_identity():
    """Naive MLA (rebuild K = [c W_uk | k_pe], V = c W_uv per head) equals
    attention over the cached rows [c | k_pe] with the absorbed query and
    V = c, followed by W_uv ("Full 路线" sections 4.2-4.3, 4.5 numerical
    check; "GQA和MLA详解" section 3)."""
    H, T, d_c, d_nope, d_R, d_v = 4, 33, 32, 8, 4, 8
    c, kpe = rnd((T, d_c), 41, 0.5), rnd((T, d_R), 42)
    qn, qr = rnd((H, d_nope), 43), rnd((H, d_R), 44)
    Wuk, Wuv = rnd((d_c, H * d_nope), 45, 0.3), rnd((d_c, H * d_v), 46, 0.3)
    scale = 1 / math.sqrt(d_nope + d_R)
    naive = npo.mla_naive_decode(c, kpe, qn, qr, Wuk, Wuv, scale)
    absorbed = npo.mla_absorbed_decode(c, kpe, qn, qr, Wuk, Wuv, scale)
    np.testing.assert_allclose(absorbed, naive, rtol=1e-12, atol=1e-13)
    # the pin discriminates: putting k_pe first in the cached row breaks it
    rows_wrong = np.concatenate([kpe, c], axis=1)
    qp = npo.mla_absorb_query(qn, qr, Wuk)
    o_lat, _ = npo.attention_fwd(qp[None, :, None], rows_wrong[None, None], c[None, None], [T], scale, False)
    wrong = np.stack([Wuv[:, h * d_v:(h + 1) * d_v].T @ o_lat[0, h, 0] for h in range(H)])
    assert not np.allclose(wrong, naive)


def test_c_oracle_mla_view_matches_numpy():
    """The C oracle on the strided MLA view (V = first 512 of 576 columns,
    same storage) agrees with the numpy oracle."""
    B, S, Hq = 2, 21, 8
    cache = rnd((B, S, 576), 47).astype(np.float32)
    q = rnd((B, Hq, 1, 576), 48).astype(np.float32)
    k = cache[:, None]
    v = cache[:, None, :, :512]
    o1, l1 = c_oracle.attention_fwd(q, k, v, [21, 9], 1 / math.sqrt(192), True, nthreads=3)
    o2, l2 = npo.attention_fwd(q, k, v, [21, 9], 1 / math.sqrt(192), True)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=1e-13, atol=1e-13)


def test_c_oracle_pairs_and_rows_agree():
    """Sampled evaluation (C oracle on listed (b,h) pairs; numpy on listed
    rows) equals the full evaluation."""
    q, k, v = rnd((2, 4, 6, 8), 49), rnd((2, 2, 10, 8), 50), rnd((2, 2, 10, 4), 51)
    full_o, full_l = npo.attention_fwd(q, k, v, [10, 7], 0.5, True)
    o, l = c_oracle.attention_fwd(q, k, v, [10, 7], 0.5, True, pairs=[(1, 3), (0, 0)])
    np.testing.assert_allclose(o[1, 3], full_o[1, 3], rtol=1e-13)
    np.testing.assert_allclose(o[0, 0], full_o[0, 0], rtol=1e-13)
    assert np.isnan(o[0, 1]).all()
    rows = [(0, 1, 0), (1, 3, 5), (1, 0, 2)]
    ro, rl = npo.attention_rows(q, k, v, [10, 7], 0.5, True, rows)
    for r, (b, h, i) in enumerate(rows):
        np.testing.assert_allclose(ro[r], full_o[b, h, i], rtol=1e-13)
        np.testing.assert_allclose(rl[r], full_l[b, h, i], rtol=1e-13)


# ----------------------------------------------------- page-printed numbers

def test_byte_model_matches_printed_tables():
    """The per-token byte counts used for the decode roofline reproduce the
    figures the pages print ("Full 路线" sections 4.4 and 4.5; "算子讲解手记
    （一）" section 3; zdabc.icu MQA article)."""
    with open(os.path.join(GOLDEN, "kv_cache_bytes.json")) as f:
        g = json.load(f)
    sh = g["mla_decode_naive_vs_absorbed"]["shape"]
    for row in g["mla_decode_naive_vs_absorbed"]["rows"]:
        naive, absorbed = npo.mla_decode_bytes(row["T"], H=sh["H"], d_nope=sh["d_nope"],
                                               d_R=sh["d_R"], d_v=sh["d_v"], d_c=sh["d_c"])
        assert int(naive / 1e6) == row["naive_MB"]  # page prints decimal MB, truncated
        assert round(absorbed / 1e6, 1 if row["absorbed_MB"] < 10 else 0) == row["absorbed_MB"]
        assert round(naive / absorbed) == row["memory_ratio"]
    for row in g["kv_bytes_per_token_per_layer"]["rows"]:
        kw = {kk: row[kk] for kk in ("H", "d_h", "G", "d_c", "d_R") if kk in row}
        assert npo.kv_bytes_per_token(row["kind"], **kw) == row["bytes"]
    cd = g["cache_dims_per_token"]
    assert npo.kv_bytes_per_token("mha", elem_bytes=1) == cd["mha_values"]
    # the p5 table counts only the latent c_kv values (no rope part), one element each
    assert npo.kv_bytes_per_token("mla", d_R=0, elem_bytes=1) == cd["mla_values"]
    assert cd["mha_values"] / cd["mla_values"] == 64  # the page's ~64x reduction
    mq = g["mqa_cache_fraction"]
    assert npo.kv_bytes_per_token("mqa", d_h=512) / npo.kv_bytes_per_token(
        "mha", H=mq["query_heads"], d_h=512) == mq["fraction"]


# ------------------------------------------------------- top-k (DSA) pins

def _topk_case(seed, B=3, Hq=8, Hkv=2, Sq=1, S=40, d=16, dv=12):
    q = rnd((B, Hq, Sq, d), seed)
    k = rnd((B, Hkv, S, d), seed + 1)
    v = rnd((B, Hkv, S, dv), seed + 2)
    return q, k, v


def test_topk_matches_sdpa_on_library_gathered_rows():
    """Attention over the selected keys equals torch SDPA (fp64, enable_gqa)
    on K/V rows picked by torch.index_select, per sequence ("带你了解Attention"
    section 5.1: attention runs over the top-k entries only)."""
    q, k, v = _topk_case(60, Sq=3)
    skv = [40, 25, 9]
    g = np.random.default_rng(61)
    n_sel = [7, 25, 1]
    idx = np.zeros((3, 25), dtype=np.int64)
    for b in range(3):
        idx[b, :n_sel[b]] = g.choice(skv[b], n_sel[b], replace=False)
    out, lse = npo.topk_attention_fwd(q, k, v, skv, idx, n_sel, 0.4)
    for b in range(3):
        sel = torch.from_numpy(idx[b, :n_sel[b]])
        kb = torch.from_numpy(k[b:b + 1]).index_select(2, sel)
        vb = torch.from_numpy(v[b:b + 1]).index_select(2, sel)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[b:b + 1]), kb, vb, scale=0.4, enable_gqa=True).numpy()
        np.testing.assert_allclose(out[b:b + 1], ref, rtol=1e-12, atol=1e-13)
        s = 0.4 * torch.from_numpy(q[b]) @ kb[0].repeat_interleave(4, dim=0).transpose(-1, -2)
        np.testing.assert_allclose(lse[b], torch.logsumexp(s, dim=-1).numpy(), rtol=1e-12)


def test_topk_all_positions_is_dense_decode():
    """Selecting every position of a sequence is ordinary decode attention
    (pinned above against SDPA)."""
    q, k, v = _topk_case(62)
    skv = [40, 3, 17]
    idx = np.zeros((3, 40), dtype=np.int64)
    for b, L in enumerate(skv):
        idx[b, :L] = np.arange(L)
    out, lse = npo.topk_attention_fwd(q, k, v, skv, idx, skv, 0.3)
    ref_o, ref_l = npo.attention_fwd(q, k, v, skv, 0.3, True)
    np.testing.assert_allclose(out, ref_o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, ref_l, rtol=1e-12, atol=1e-13)


def test_topk_selection_order_and_union():
    """The order of the selected positions does not matter, and attention over
    a union of two disjoint selections is the LSE-weighted merge of the two."""
    q, k, v = _topk_case(63, B=1)
    idx = np.array([[5, 31, 2, 17, 39, 0, 22, 8]])
    a_o, a_l = npo.topk_attention_fwd(q, k, v, [40], idx, [8], 0.5)
    b_o, b_l = npo.topk_attention_fwd(q, k, v, [40], idx[:, ::-1].copy(), [8], 0.5)
    np.testing.assert_allclose(a_o, b_o, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(a_l, b_l, rtol=1e-13, atol=1e-14)
    p_o, p_l = npo.topk_attention_fwd(q, k, v, [40], idx[:, :3].copy(), [3], 0.5)
    r_o, r_l = npo.topk_attention_fwd(q, k, v, [40], idx[:, 3:].copy(), [5], 0.5)
    m_o, m_l = npo.split_combine(np.stack([p_o, r_o]), np.stack([p_l, r_l]))
    np.testing.assert_allclose(m_o, a_o, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(m_l, a_l, rtol=1e-13, atol=1e-14)


def test_topk_single_repeated_and_empty():
    """One selected key: out is its value row, lse its score.  The same key
    listed twice: the same row, lse + ln 2.  Nothing selected: 0 and -inf."""
    q, k, v = _topk_case(64, B=3, Hq=2, Hkv=1)
    idx = np.array([[13, 0], [13, 13], [0, 0]])
    out, lse = npo.topk_attention_fwd(q, k, v, [40, 40, 40], idx, [1, 2, 0], 0.25)
    for h in range(2):
        s = 0.25 * float(q[0, h, 0] @ k[0, 0, 13])
        np.testing.assert_array_equal(out[0, h, 0], v[0, 0, 13])
        assert abs(lse[0, h, 0] - s) < 1e-13
        s1 = 0.25 * float(q[1, h, 0] @ k[1, 0, 13])
        np.testing.assert_allclose(out[1, h, 0], v[1, 0, 13], rtol=1e-15, atol=1e-15)
        assert abs(lse[1, h, 0] - (s1 + math.log(2))) < 1e-13
    assert (out[2] == 0).all() and np.isneginf(lse[2]).all()


def test_topk_rejects_positions_outside_the_sequence():
    q, k, v = _topk_case(65, B=1)
    with pytest.raises(ValueError):
        npo.topk_attention_fwd(q, k, v, [10], np.array([[3, 10]]), [2], 0.5)
    with pytest.raises(ValueError):
        npo.topk_attention_fwd(q, k, v, [10], np.array([[-1, 2]]), [2], 0.5)


# --------------------------------------------- the two oracles, randomised


@settings(max_examples=60, deadline=None)
@given(B=st.integers(1, 3), Hkv=st.integers(1, 3), G=st.integers(1, 4), Sq=st.integers(1, 9),
       d=st.sampled_from([1, 3, 8, 16]), dv=st.sampled_from([1, 5, 8]), causal=st.booleans(),
       data=st.data())
def test_numpy_and_c_oracles_agree(B, Hkv, G, Sq, d, dv, causal, data):
    """The numpy and C oracles share no code; on random ragged shapes
    (lengths 0..20, Sq above and below them, any grouping) they must agree
    to rounding, including which rows are empty."""
    skv = data.draw(st.lists(st.integers(0, 20), min_size=B, max_size=B))
    S = max(max(skv), 1)
    seed = data.draw(st.integers(0, 10_000))
    q, k, v = rnd((B, Hkv * G, Sq, d), seed), rnd((B, Hkv, S, d), seed + 1), rnd((B, Hkv, S, dv), seed + 2)
    scale = data.draw(st.sampled_from([0.1, 0.5, 1.3]))
    o1, l1 = npo.attention_fwd(q, k, v, skv, scale, causal)
    o2, l2 = c_oracle.attention_fwd(q, k, v, skv, scale, causal, nthreads=2)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    assert (np.isneginf(l1) == np.isneginf(l2)).all()
    fin = np.isfinite(l1)
    np.testing.assert_allclose(l1[fin], l2[fin], rtol=1e-12, atol=1e-13)
