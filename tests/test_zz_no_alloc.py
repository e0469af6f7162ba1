"""attn_fwd_noalloc: the entry point for callers that cannot allocate device
memory (e.g. a plugin whose host framework owns all device memory, or a
latency-critical loop that cannot afford cudaMalloc's implicit device
synchronisation).  It runs the same kernels with the same launch plan as
attn_fwd, whose workspace the caller provides, so its results must be
bitwise the same; it takes its scratch from the buffer built into the
library instead.

This file is collected last on purpose, so that a run stopping at its first
failure has already run every other test.  It does not depend on state left
by other tests and passes when run alone in a fresh process.
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


def _both(case):
    """Run attn_fwd (caller workspace) and attn_fwd_noalloc (built-in
    scratch) on the same inputs; return both (out, lse)."""
    from attention_mqa_gqa_b200 import binding

    w, inp = case
    dev = to_device(inp)
    ref_out, ref_lse = binding.attention(dev["q"], dev["k"], dev["v"], dev["skv"],
                                         dev["max_skv"], w.scale, w.causal)
    out = torch.full_like(ref_out, float("nan"))
    lse = torch.full_like(ref_lse, float("nan"))
    binding.attn_fwd_noalloc(dev["q"], dev["k"], dev["v"], out, dev["skv"], dev["max_skv"],
                             w.scale, w.causal, lse)
    torch.cuda.synchronize()
    assert binding.last_device_error() == binding.ATTN_OK
    return (out, lse), (ref_out, ref_lse)


def _check(case):
    (o, l), (ro, rl) = _both(case)
    # same kernels, same plan: the scratch location must not change a bit
    assert torch.equal(o, ro) and torch.equal(l, rl)
    # and the result is the attention the oracle computes
    w, inp = case
    ref_o, ref_l = oracle_full(w, inp)
    compare(o, l, ref_o, ref_l, f"noalloc {w.name}")


def test_noalloc_matches_attn_fwd_twice_in_a_row():
    """Two calls in a row with different problems: the second must not be
    affected by what the first left in the shared scratch buffer."""
    first = wl.make_case(6, 16, 1, 1, [3000, 129, 1, 4500, 777, 2048], 512, 512, seed=31)
    second = wl.make_case(5, 64, 8, 1, [1000, 4096, 300, 17, 2500], 128, 128, seed=32)
    for case in (first, second):
        _check(case)


def test_noalloc_mla_decode_and_prefill():
    """The SM-pair MLA decode (scratch in use) and a causal prefill, which
    needs no scratch at all (the call passes none to the kernels)."""
    _check(wl.make_case(3, 128, 1, 1, [900, 257, 2], 576, 512, mla=True, seed=33,
                        scale=192 ** -0.5))
    _check(wl.make_case(1, 8, 2, 200, [200], 128, 128, causal=True, seed=34))


def test_noalloc_refuses_problems_larger_than_its_scratch():
    from attention_mqa_gqa_b200 import binding

    # MLA decode at 64 x 16384 keys needs ~67 MB of partials: more than the buffer.
    B, Hq, S = 64, 128, 16384
    need = binding.workspace_bytes(B, Hq, 1, 1, S, 576, 512)
    assert need > binding.NOALLOC_SCRATCH_BYTES
    q = torch.zeros(B, Hq, 1, 576, dtype=torch.bfloat16, device="cuda")
    cache = torch.zeros(B, 1, 128, 576, dtype=torch.bfloat16, device="cuda")  # never read
    out = torch.empty(B, Hq, 1, 512, dtype=torch.bfloat16, device="cuda")
    skv = torch.ones(B, dtype=torch.int32, device="cuda")
    with pytest.raises(binding.AttnError) as e:
        binding.attn_fwd_noalloc(q, cache, cache[..., :512], out, skv, S, 0.07, True)
    assert e.value.status == binding.ATTN_EWORKSPACE
