"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small cases and the full-size workloads compare every output element and
LSE.  Tolerance:
|gpu - oracle| <= 1e-2 + 1e-2*|oracle| per element, |dLSE| <= 1e-3.
"""
import math

import numpy as np
import pytest
import torch

from attention_mqa_gqa_b200 import workloads as wl
from tests.helpers import compare, oracle_full, run_gpu, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from attention_mqa_gqa_b200 import binding, build

    build.build()
    binding.load()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _poison_past_length(inp):
    """Set every cache row at or past its sequence's length to NaN.  Those
    rows are not part of the problem (a cache allocated for max_skv keys
    holds whatever memory had there), so the result must not change."""
    for b, L in enumerate(inp["skv"].tolist()):
        if "cache" in inp:
            inp["cache"][b, L:] = float("nan")
        else:
            inp["k"][b, :, L:] = float("nan")
            inp["v"][b, :, L:] = float("nan")


def _case(B, Hq, Hkv, Sq, skv, dk, dv, dtype=torch.bfloat16, causal=True, mla=False, seed=0,
          max_skv=None, scale=None, poison=False):
    w, inp = wl.make_case(B, Hq, Hkv, Sq, skv, dk, dv, dtype=dtype, causal=causal, mla=mla,
                          seed=seed, max_skv=max_skv, scale=scale)
    if poison:
        _poison_past_length(inp)
    dev = to_device(inp)
    out, lse = run_gpu(w, dev)
    ref_o, ref_l = oracle_full(w, inp)
    return compare(out, lse, ref_o, ref_l, what=w.name)


# ------------------------------------------------------------------ decode

@pytest.mark.parametrize("Hq,Hkv", [(8, 1), (16, 2), (4, 4), (32, 2), (40, 2)])
def test_decode_d128(Hq, Hkv):
    _case(3, Hq, Hkv, 1, [1, 129, 700], 128, 128, seed=Hq + Hkv)


@pytest.mark.parametrize("skv", [[1], [127], [128], [129], [255, 256, 257], [3000, 17, 1024]])
def test_decode_d128_ragged(skv):
    _case(len(skv), 8, 1, 1, skv, 128, 128, seed=sum(skv))


@pytest.mark.parametrize("Hq,skv", [(16, [1, 129, 700, 2049]), (4, [300, 5]), (16, [4097])])
def test_decode_mqa_d512(Hq, skv):
    _case(len(skv), Hq, 1, 1, skv, 512, 512, seed=7)


@pytest.mark.parametrize("Hq,skv", [(128, [1, 200, 1500]), (16, [513, 64]), (64, [2000])])
def test_decode_mla(Hq, skv):
    _case(len(skv), Hq, 1, 1, skv, 576, 512, mla=True, seed=11, scale=1 / math.sqrt(192))


@pytest.mark.parametrize("B,Hq,Hkv,Sq,skv,dk,causal", [
    (3, 16, 2, 4, [1000, 3, 129], 128, True),    # skv < Sq: early queries see nothing
    (2, 16, 2, 2, [700, 2], 128, True),
    (2, 16, 2, 8, [4097, 300], 128, True),
    (2, 16, 1, 4, [2000, 5], 512, True),
    (2, 16, 2, 4, [777, 1], 128, False),
    (2, 4, 4, 16, [1500, 20], 128, True),        # G = 1: 16 queries of one head per CTA
])
def test_decode_extend(B, Hq, Hkv, Sq, skv, dk, causal):
    """Sq > 1 queries against a cache (extend / speculative decoding) on the
    split-KV decode path, bottom-right causal alignment."""
    _case(B, Hq, Hkv, Sq, skv, dk, dk, causal=causal, seed=40 + Sq)


def test_decode_fp16():
    _case(2, 16, 1, 1, [333, 1000], 512, 512, dtype=torch.float16, seed=3)


def test_decode_zero_length_sequence():
    _case(3, 16, 1, 1, [0, 300, 0], 512, 512, seed=5, max_skv=300)


@pytest.mark.parametrize("case", ["mqa_d512", "gqa_extend", "mla"])
def test_decode_two_phase_entry_points(case):
    """attn_decode_partial followed by attn_decode_combine (the separate
    merge kernel) gives the attention too; attn_fwd merges inside the split
    kernel instead."""
    from attention_mqa_gqa_b200 import binding

    if case == "mqa_d512":
        w, inp = wl.make_case(3, 16, 1, 1, [2000, 0, 777], 512, 512, seed=71)
    elif case == "gqa_extend":
        w, inp = wl.make_case(2, 16, 2, 4, [300, 3], 128, 128, seed=72)
    else:
        w, inp = wl.make_case(2, 128, 1, 1, [3000, 300], 576, 512, mla=True, seed=73,
                              scale=192 ** -0.5)
    dev = to_device(inp)
    q, k, v = dev["q"], dev["k"], dev["v"]
    B, Hq, Sq, dk = q.shape
    out = torch.full((B, Hq, Sq, v.shape[-1]), float("nan"), dtype=q.dtype, device="cuda")
    lse = torch.full((B, Hq, Sq), float("nan"), dtype=torch.float32, device="cuda")
    n = binding.workspace_bytes(B, Hq, k.shape[1], Sq, dev["max_skv"], dk, v.shape[-1])
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    st = lambda t: binding.Strides(t.stride(0), t.stride(1), t.stride(2))
    for entry in ("attn_decode_partial", "attn_decode_combine"):
        rc = binding.fwd_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                             lse.data_ptr(), B, Hq, k.shape[1], Sq, dev["skv"].data_ptr(),
                             dev["max_skv"], dk, v.shape[-1], w.scale, w.causal,
                             binding.dtype_code(q.dtype), st(q), st(k), st(v), st(out),
                             ws.data_ptr(), n, torch.cuda.current_stream().cuda_stream,
                             entry=entry)
        assert rc == binding.ATTN_OK
    torch.cuda.synchronize()
    assert binding.last_device_error() == binding.ATTN_OK
    ref_o, ref_l = oracle_full(w, inp)
    compare(out, lse, ref_o, ref_l, f"two-phase {case}")


def test_decode_strided_views():
    """q/out as views with padded strides; K/V as slices of a wider buffer."""
    from attention_mqa_gqa_b200 import binding
    from oracle import c_oracle

    g = torch.Generator().manual_seed(9)
    B, Hq, Hkv, S, d = 2, 16, 2, 400, 128
    qbig = torch.randn(B, Hq, 1, d + 64, generator=g).to(torch.bfloat16)
    kbig = torch.randn(B, Hkv, S, d + 128, generator=g).to(torch.bfloat16)
    vbig = torch.randn(B, Hkv, S, d + 64, generator=g).to(torch.bfloat16)
    q, k, v = qbig[..., 8:8 + d], kbig[..., 64:64 + d], vbig[..., :d]
    skv = torch.tensor([400, 211], dtype=torch.int32)
    qd, kd, vd = qbig.cuda()[..., 8:8 + d], kbig.cuda()[..., 64:64 + d], vbig.cuda()[..., :d]
    outbig = torch.zeros(B, Hq, 1, d + 32, dtype=torch.bfloat16, device="cuda")
    out = outbig[..., 16:16 + d]
    lse = torch.empty(B, Hq, 1, device="cuda")
    ws = torch.empty(binding.workspace_bytes(B, Hq, Hkv, 1, S, d, d), dtype=torch.uint8, device="cuda")
    binding.attn_fwd(qd, kd, vd, out, skv.cuda(), S, 0.1, True, lse, ws)
    torch.cuda.synchronize()
    ref_o, ref_l = c_oracle.attention_fwd(q, k, v, skv.tolist(), 0.1, True)
    compare(out, lse, ref_o, ref_l, "strided decode")
    assert (outbig[..., :16] == 0).all() and (outbig[..., 16 + d:] == 0).all()


# ----------------------------------------------------------------- prefill

@pytest.mark.parametrize("Sq,skv,causal", [(200, 200, True), (200, 200, False), (128, 128, True),
                                           (257, 257, True), (130, 300, True), (1, 1, True)])
def test_prefill_d128(Sq, skv, causal):
    if Sq == 1:
        pytest.skip("Sq == 1 takes the decode path")
    _case(1, 4, 2, Sq, [skv], 128, 128, causal=causal, seed=Sq)


def test_prefill_d128_varlen_bottom_right():
    """Two sequences with fewer keys than queries in one: bottom-right
    alignment leaves the first rows with no visible key (out 0, lse -inf)."""
    _case(2, 8, 1, 150, [300, 100], 128, 128, causal=True, seed=21, max_skv=300)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_prefill_d512(dtype):
    _case(1, 16, 1, 300, [300], 512, 512, dtype=dtype, causal=True, seed=4)


def test_prefill_d512_noncausal_ragged():
    _case(2, 4, 1, 129, [129, 129], 512, 512, causal=False, seed=6)


@pytest.mark.parametrize("Hq,Hkv,Sq,skv,causal", [(8, 8, 300, [300], True),
                                                  (4, 2, 129, [200], True),
                                                  (8, 8, 257, [257], False)])
def test_prefill_mla_expanded(Hq, Hkv, Sq, skv, causal):
    """MLA prefill in the expanded (MHA) form ("带你了解Attention" section 4.4:
    prefill runs as ordinary attention on reconstructed K, V): q/k rows of
    192 = 128 + 64 (rope) columns -- an odd number of 64-column chunks --
    and v rows of 128, scale 1/sqrt(192)."""
    _case(len(skv), Hq, Hkv, Sq, skv, 192, 128, causal=causal, seed=30 + Sq,
          scale=1 / math.sqrt(192))


def test_prefill_mqa_tiny_workload():
    """The MQA d=512 fp16 prefill workload (B=1, Hq=16, S=128) in full."""
    w = wl.WORKLOADS["mqa_prefill_tiny"]
    inp = wl.make_inputs(w)
    out, lse = run_gpu(w, to_device(inp))
    ref_o, ref_l = oracle_full(w, inp)
    compare(out, lse, ref_o, ref_l, w.name)


# --------------------------------------- cache rows past a sequence's end

@pytest.mark.parametrize("B,Hq,Hkv,Sq,skv,max_skv,dk,dv,mla", [
    (3, 16, 2, 1, [1, 129, 700], 1024, 128, 128, False),     # GQA decode
    (3, 16, 1, 1, [1, 300, 2049], 2100, 512, 512, False),    # MQA d=512 decode
    (3, 128, 1, 1, [1, 200, 1500], 1600, 576, 512, True),    # MLA pair decode
    (2, 16, 2, 4, [1000, 3], 1100, 128, 128, False),         # extend, Sq = 4
])
def test_decode_ignores_rows_past_length(B, Hq, Hkv, Sq, skv, max_skv, dk, dv, mla):
    """NaN in every cache row at or past skv[b] (as in a cache allocated for
    max_skv keys and filled as it grows) must not reach the output."""
    _case(B, Hq, Hkv, Sq, skv, dk, dv, mla=mla, seed=80 + Sq, max_skv=max_skv, poison=True,
          scale=1 / math.sqrt(192) if mla else None)


@pytest.mark.parametrize("B,Hq,Hkv,Sq,skv,max_skv,dk,dv", [
    (2, 8, 1, 150, [300, 100], 320, 128, 128),     # d=128, varlen, bottom-right
    (2, 16, 1, 129, [129, 129], 200, 512, 512),    # d=512, SM pairs (even G)
    (1, 3, 1, 129, [150], 256, 512, 512),          # d=512, one CTA per tile (odd G)
    (1, 4, 2, 129, [200], 256, 192, 128),          # expanded MLA, d_k 192 / d_v 128
    (1, 4, 2, 100, [100], 256, 128, 128),          # shorter than one key tile
])
def test_prefill_ignores_rows_past_length(B, Hq, Hkv, Sq, skv, max_skv, dk, dv):
    _case(B, Hq, Hkv, Sq, skv, dk, dv, seed=90 + Sq, max_skv=max_skv, poison=True)


# ------------------------------------------------------------- determinism

def test_bitwise_reproducible():
    w, inp = wl.make_case(4, 16, 1, 1, [5000, 100, 2000, 7000], 512, 512, seed=13)
    dev = to_device(inp)
    a, la = run_gpu(w, dev)
    b, lb = run_gpu(w, dev)
    assert torch.equal(a, b) and torch.equal(la, lb)
    w, inp = wl.make_case(1, 4, 1, 600, [600], 128, 128, seed=14)
    dev = to_device(inp)
    a, la = run_gpu(w, dev)
    b, lb = run_gpu(w, dev)
    assert torch.equal(a, b) and torch.equal(la, lb)


# ------------------------------------------------------- full-size workloads

def _full_size(name):
    from oracle import c_oracle

    w = wl.WORKLOADS[name]
    inp = wl.make_inputs(w)
    out, lse = run_gpu(w, to_device(inp))
    # Every output element and LSE against the fp64 C oracle on all host
    # threads: decode batches take seconds; the prefill batches (0.55-1.1
    # TFLOP of fp64 work) take about a minute each.  At full size the
    # prefill kernel walks its work in blocks of heads (expanded MLA: 15 of
    # 128 heads per block, the last block partial) and heavy q tiles first,
    # which only a whole-output comparison covers.
    ref_o, ref_l = c_oracle.attention_fwd(inp["q"], inp["k"], inp["v"], inp["skv"].tolist(),
                                          w.scale, w.causal)
    compare(out, lse, ref_o, ref_l, f"{name} (every element)")


@pytest.mark.parametrize("name", ["mqa_decode", "gqa_decode", "mla_decode", "mqa_prefill",
                                  "gqa_prefill", "mla_prefill", "gqa_extend"])
def test_full_workload(name):
    """Each workload at its benchmark size, launched as bench.py launches it,
    checked on every output element."""
    _full_size(name)
