"""The error path of the device-side waits, exercised without any fault.

Every mbarrier wait in the kernels is bounded.  With the bound set far
below the kernels' normal waiting times (1 ns: a wait that is not
satisfied within its first few hundred polls gives up), each launch takes
its abort path: the role that gave up raises the CTA's abort flag, the
other roles leave their loops, issued copies and MMAs drain, TMEM is freed
and the kernel returns.  The host must then read ATTN_ETIMEOUT from
attn_last_device_error, and the context must stay usable: with the default
bound restored, the same call gives the oracle's result and reports OK.
"""
import pytest
import torch

from attention_mqa_gqa_b200 import workloads as wl
from tests.helpers import compare, oracle_full, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from attention_mqa_gqa_b200 import binding, build

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    binding.load()
    yield
    binding.set_wait_timeout_ns(0)


CASES = {
    "decode_mqa_d512": dict(B=4, Hq=16, Hkv=1, Sq=1, skv=[3000, 700, 5000, 129], d_k=512, d_v=512),
    "decode_mla": dict(B=2, Hq=128, Hkv=1, Sq=1, skv=[4100, 900], d_k=576, d_v=512, mla=True,
                       scale=192 ** -0.5),
    "prefill_gqa_d128": dict(B=1, Hq=8, Hkv=2, Sq=700, skv=[700], d_k=128, d_v=128),
    "prefill_mqa_d512": dict(B=1, Hq=4, Hkv=1, Sq=384, skv=[384], d_k=512, d_v=512),
}


@pytest.mark.parametrize("name", list(CASES))
def test_wait_timeout_reports_and_recovers(name):
    from attention_mqa_gqa_b200 import binding

    c = dict(CASES[name])
    w, inp = wl.make_case(c.pop("B"), c.pop("Hq"), c.pop("Hkv"), c.pop("Sq"), c.pop("skv"),
                          c.pop("d_k"), c.pop("d_v"), seed=21, **c)
    dev = to_device(inp)
    assert binding.last_device_error() == binding.ATTN_OK  # nothing pending

    prev = binding.set_wait_timeout_ns(1)
    try:
        binding.attention(dev["q"], dev["k"], dev["v"], dev["skv"], dev["max_skv"], w.scale,
                          w.causal)
        status = binding.last_device_error()  # synchronises the stream
    finally:
        binding.set_wait_timeout_ns(prev)
    assert status == binding.ATTN_ETIMEOUT, binding.status_str(status)
    assert binding.last_device_error() == binding.ATTN_OK  # the word was read and cleared

    out, lse = binding.attention(dev["q"], dev["k"], dev["v"], dev["skv"], dev["max_skv"],
                                 w.scale, w.causal)
    torch.cuda.synchronize()
    assert binding.last_device_error() == binding.ATTN_OK
    ref_o, ref_l = oracle_full(w, inp)
    compare(out, lse, ref_o, ref_l, f"{name} after a timed-out launch")
