"""Top-k sparse decode (DSA style, "带你了解Attention" section 5.1): the rows
at caller-selected positions are gathered (attn_gather_rows) and attention
runs over them (attn_fwd), or, for absorbed MLA, the decode kernel gathers
them itself (attn_topk_fwd); both compared with the oracle's attention over
the selected subset, and with each other bitwise.  Also: the gathered rows
are bitwise copies, ragged and empty selections, a position outside its
sequence reported as ATTN_EINDEX by both paths, and every output of the
full-size 2048-of-16K..48K MLA workload."""
import math

import pytest
import torch

from attention_mqa_gqa_b200 import workloads as wl
from tests.helpers import compare, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from attention_mqa_gqa_b200 import binding, build

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    binding.load()


CASES = {
    "mla_latent": dict(Hq=128, Hkv=1, dk=576, dv=512, mla=True, scale=1 / math.sqrt(192)),
    "mqa_d512": dict(Hq=16, Hkv=1, dk=512, dv=512, mla=False, scale=None),
    "gqa_d128": dict(Hq=16, Hkv=4, dk=128, dv=128, mla=False, scale=None),
}


def _run(name, skv, topk, seed, n_sel_override=None):
    from attention_mqa_gqa_b200 import binding
    from oracle import attention as npo

    c = CASES[name]
    B = len(skv)
    w, inp = wl.make_case(B, c["Hq"], c["Hkv"], 1, skv, c["dk"], c["dv"], mla=c["mla"],
                          scale=c["scale"], seed=seed)
    idx, n_sel = wl.make_selection(skv, topk, torch.Generator().manual_seed(seed + 1))
    if n_sel_override is not None:
        n_sel = torch.tensor(n_sel_override, dtype=torch.int32)
    dev = to_device(inp)
    sc = {}
    out, lse = binding.topk_attention(dev["q"], dev["k"], None if c["mla"] else dev["v"],
                                      idx.cuda(), n_sel.cuda(), dev["skv"], w.scale,
                                      d_v=c["dv"], scratch=sc, fused=False)
    torch.cuda.synchronize()
    assert binding.last_device_error() == binding.ATTN_OK
    if c["mla"]:  # the one-pass path: the same kernel on the same rows, bit for bit
        out_f, lse_f = binding.topk_attention(dev["q"], dev["k"], None, idx.cuda(), n_sel.cuda(),
                                              dev["skv"], w.scale, d_v=c["dv"])
        torch.cuda.synchronize()
        assert binding.last_device_error() == binding.ATTN_OK
        assert torch.equal(out_f, out) and torch.equal(lse_f, lse)
    # the gathered rows are bitwise copies of the selected cache rows
    kg = sc["k"].cpu()
    assert torch.equal(sc["len"].cpu(), n_sel)
    for b in range(B):
        n = int(n_sel[b])
        sel = idx[b, :n].long()
        assert torch.equal(kg[b, :, :n], inp["k"][b][:, sel])
        if not c["mla"]:
            assert torch.equal(sc["v"].cpu()[b, :, :n], inp["v"][b][:, sel])
    ref_o, ref_l = npo.topk_attention_fwd(inp["q"], inp["k"], inp["v"], skv, idx, n_sel.tolist(),
                                          w.scale)
    return compare(out, lse, ref_o, ref_l, f"topk {name}")


@pytest.mark.parametrize("name", list(CASES))
def test_topk_decode(name):
    # 256 of 3000 / all 200 (fewer than topk) / 256 of 5000 / an empty sequence
    _run(name, [3000, 200, 5000, 0], 256, seed=70)


@pytest.mark.parametrize("name", ["mla_latent", "gqa_d128"])
def test_topk_ragged_k(name):
    """topk not a multiple of the 128-row tiles; one selected key; n_sel
    below the number of filled slots."""
    _run(name, [4000, 900, 77], 300, seed=71, n_sel_override=[300, 1, 40])


def test_topk_position_outside_sequence_reports_eindex():
    from attention_mqa_gqa_b200 import binding

    B, d = 2, 576
    src = torch.randn(B, 1, 64, d, device="cuda").to(torch.bfloat16)
    dst = torch.full((B, 1, 8, d), 7.0, device="cuda", dtype=torch.bfloat16)
    idx = torch.tensor([[0, 5, 63, 2, 0, 0, 0, 0], [1, 64, 3, 0, 0, 0, 0, 0]],
                       dtype=torch.int32, device="cuda")
    n_sel = torch.tensor([4, 3], dtype=torch.int32, device="cuda")
    skv = torch.tensor([64, 64], dtype=torch.int32, device="cuda")
    dlen = torch.empty(B, dtype=torch.int32, device="cuda")
    binding.gather_rows(src, dst, idx, n_sel, skv, dlen)
    assert binding.last_device_error() == binding.ATTN_EINDEX
    torch.cuda.synchronize()
    assert torch.equal(dst[0, 0, :4], src[0, 0, [0, 5, 63, 2]])
    assert torch.equal(dst[1, 0, 0], src[1, 0, 1]) and (dst[1, 0, 1] == 0).all()
    assert torch.equal(dst[1, 0, 2], src[1, 0, 3])
    assert (dst[:, :, 4:].float() == 7.0).all() and (dst[1, :, 3:].float() == 7.0).all()
    assert dlen.tolist() == [4, 3]


def test_topk_fused_position_outside_sequence_reports_eindex():
    """attn_topk_fwd reads a position outside its sequence as a zero row (as
    the gather pass writes it) and reports ATTN_EINDEX."""
    from attention_mqa_gqa_b200 import binding

    B, Hq, S = 2, 128, 300
    g = torch.Generator().manual_seed(5)
    q = torch.randn(B, Hq, 1, 576, generator=g).to(torch.bfloat16).cuda()
    cache = torch.randn(B, 1, S, 576, generator=g).to(torch.bfloat16).cuda()
    idx = torch.tensor([[0, 5, 299, 2, 7, 9], [1, 300, 3, -1, 0, 0]], dtype=torch.int32,
                       device="cuda")
    n_sel = torch.tensor([4, 4], dtype=torch.int32, device="cuda")
    skv = torch.tensor([S, S], dtype=torch.int32, device="cuda")
    ref, ref_lse = binding.topk_attention(q, cache, None, idx, n_sel, skv, 0.07, d_v=512,
                                          fused=False)
    assert binding.last_device_error() == binding.ATTN_EINDEX
    out, lse = binding.topk_attention(q, cache, None, idx, n_sel, skv, 0.07, d_v=512)
    assert binding.last_device_error() == binding.ATTN_EINDEX
    torch.cuda.synchronize()
    assert torch.equal(out, ref) and torch.equal(lse, ref_lse)


def test_full_workload():
    """mla_topk_decode (B=64, 128 heads, 2048 of 16K-48K positions): every
    output element against the oracle."""
    from attention_mqa_gqa_b200 import binding
    from oracle import attention as npo

    w = wl.WORKLOADS["mla_topk_decode"]
    inp = wl.make_inputs(w)
    dev = to_device(inp)
    out, lse = binding.topk_attention(dev["q"], dev["k"], None, inp["idx"].cuda(),
                                      inp["n_sel"].cuda(), dev["skv"], w.scale, d_v=w.d_v)
    torch.cuda.synchronize()
    assert binding.last_device_error() == binding.ATTN_OK
    ref_o, ref_l = npo.topk_attention_fwd(inp["q"], inp["k"], inp["v"], inp["skv"].tolist(),
                                          inp["idx"], inp["n_sel"].tolist(), w.scale)
    compare(out, lse, ref_o, ref_l, "mla_topk_decode (every element)")
