"""attn_cache_append: the new token's rows land at position skv[b] of the
cache (bitwise), skv advances, and a decode step enqueued after it on the
same stream attends over the new key (compared with the oracle on the
cache updated on the host).  A sequence that is already full is left
unchanged and reported as ATTN_EOVERFLOW."""
import math

import pytest
import torch

from attention_mqa_gqa_b200 import workloads as wl
from tests.helpers import compare, oracle_full, run_gpu, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from attention_mqa_gqa_b200 import binding, build

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    binding.load()


CASES = {
    "mqa_d512": dict(Hq=16, Hkv=1, dk=512, dv=512, mla=False, scale=None),
    "gqa_d128": dict(Hq=16, Hkv=4, dk=128, dv=128, mla=False, scale=None),
    "mla_latent": dict(Hq=128, Hkv=1, dk=576, dv=512, mla=True, scale=1 / math.sqrt(192)),
}


def _new_rows(B, Hkv, d, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(B, Hkv, 1, d, generator=g).to(torch.bfloat16)


def _appended(inp, k_new, v_new, skv, max_skv, mla):
    """The host-side expectation: the same inputs with the new rows written
    at each sequence's length (when there is room) and lengths advanced."""
    out = dict(inp)
    new_skv = skv.clone()
    if mla:
        cache = inp["cache"].clone()
        for b in range(cache.shape[0]):
            if skv[b] < max_skv:
                cache[b, skv[b]] = k_new[b, 0, 0]
                new_skv[b] += 1
        B, S, dk = cache.shape
        out["cache"] = cache
        out["k"] = cache.view(B, 1, S, dk)
        out["v"] = cache.view(B, 1, S, dk)[..., : inp["v"].shape[-1]]
    else:
        k, v = inp["k"].clone(), inp["v"].clone()
        for b in range(k.shape[0]):
            if skv[b] < max_skv:
                k[b, :, skv[b]] = k_new[b, :, 0]
                v[b, :, skv[b]] = v_new[b, :, 0]
                new_skv[b] += 1
        out["k"], out["v"] = k, v
    out["skv"] = new_skv
    return out


def _run(name, skv, max_skv, expect_status):
    from attention_mqa_gqa_b200 import binding

    c = CASES[name]
    B = len(skv)
    w, inp = wl.make_case(B, c["Hq"], c["Hkv"], 1, skv, c["dk"], c["dv"], mla=c["mla"],
                          scale=c["scale"], seed=50, max_skv=max_skv)
    k_new = _new_rows(B, c["Hkv"], c["dk"], 51)
    v_new = None if c["mla"] else _new_rows(B, c["Hkv"], c["dv"], 52)
    dev = to_device(inp)
    binding.cache_append(dev["k"], None if c["mla"] else dev["v"], k_new.cuda(),
                         None if c["mla"] else v_new.cuda(), dev["skv"])
    status = binding.last_device_error()
    assert status == expect_status, binding.status_str(status)

    exp = _appended(inp, k_new, v_new, inp["skv"], max_skv, c["mla"])
    assert torch.equal(dev["skv"].cpu(), exp["skv"])
    if c["mla"]:
        assert torch.equal(dev["cache"].cpu(), exp["cache"])
    else:
        assert torch.equal(dev["k"].cpu(), exp["k"]) and torch.equal(dev["v"].cpu(), exp["v"])

    # the decode step after the append sees the new key
    w2 = w.scaled(skv_lo=int(exp["skv"].min()), skv_hi=int(exp["skv"].max()))
    out, lse = run_gpu(w2, dev)
    ref_o, ref_l = oracle_full(w2, exp)
    compare(out, lse, ref_o, ref_l, f"{name} after append")


@pytest.mark.parametrize("name", list(CASES))
def test_append_then_decode(name):
    _run(name, [100, 0, 2047, 700], 2048, 0)


def test_append_full_sequence_reports_overflow():
    from attention_mqa_gqa_b200 import binding

    _run("gqa_d128", [300, 300, 17], 300, binding.ATTN_EOVERFLOW)
