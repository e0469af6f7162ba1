"""Host-side checks of the C ABI (no GPU): the library builds and loads,
exports every entry point the header declares, plans correctly, and rejects
bad arguments before anything reaches the device."""
import ctypes
import os
import re

import pytest

from attention_mqa_gqa_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn_b200.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z_]+)\s*\(", text)))


def test_header_declarations_are_exported(lib):
    names = declared_functions()
    assert set(names) == set(binding.EXPORTS), names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in the header but not exported"


def test_noalloc_scratch_size_matches_header():
    """The binding's copy of the built-in scratch size is the header's."""
    m = re.search(r"#define\s+ATTN_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)",
                  open(HEADER).read())
    assert m, "ATTN_NOALLOC_SCRATCH_BYTES not found in the header"
    assert binding.NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))


def test_status_strings(lib):
    for code in range(8):
        assert binding.status_str(code) and binding.status_str(code) != "unknown status"
    assert binding.version().count(".") == 2


def test_plan_decode_invariants(lib):
    for (B, Hq, Hkv, S, dk, dv) in [(32, 16, 1, 8192, 512, 512), (64, 64, 8, 4096, 128, 128),
                                    (64, 128, 1, 16384, 576, 512), (1, 8, 8, 1, 128, 128),
                                    (3, 40, 2, 1000, 128, 128)]:
        pl = binding.plan(B, Hq, Hkv, 1, S, dk, dv, num_sms=148)
        G = Hq // Hkv
        assert pl["path"] == 1
        # MLA runs on pairs of SMs (one cluster of two CTAs per key range)
        # that together hold all 128 heads; the others 16 heads per CTA
        assert pl["heads_per_cta"] == (128 if dk == 576 else 16)
        assert pl["head_blocks"] == -(-G // pl["heads_per_cta"])
        ctas_per_range = 2 if dk == 576 else 1
        ctas_per_sm = 2 if dk == 128 else 1
        assert pl["kv_ranges"] == max(1, 148 * ctas_per_sm // ctas_per_range // pl["head_blocks"])
        assert pl["grid_ctas"] == pl["kv_ranges"] * pl["head_blocks"] * ctas_per_range
        assert pl["partials"] == pl["kv_ranges"] + B * Hkv
        n = pl["partials"] * G
        r256 = lambda x: (x + 255) // 256 * 256
        # partial outputs, partial LSEs, then the in-kernel merge's arrival
        # counters: one per (unit, head block), per CTA of the pair for MLA
        counters = B * Hkv * pl["head_blocks"] * (2 if dk == 576 else 1)
        assert pl["workspace_bytes"] == r256(n * dv * 4) + r256(n * 4) + r256(counters * 4)


def _ranges_pieces(skv, Hkv, R):
    """Independent model of the decode schedule: concatenated tiles of the
    (b, kvh) units cut into R equal ranges; pieces = nonempty overlaps."""
    tiles = [(L + 127) // 128 for L in skv]
    units = [(b, k, tiles[b]) for b in range(len(skv)) for k in range(Hkv)]
    T = sum(t for _, _, t in units)
    R = min(R, T)  # only ranges that hold at least one tile are used
    bounds = [r * T // R for r in range(R + 1)] if R else [0]
    pieces, start = [], 0
    for u, (b, k, t) in enumerate(units):
        for r in range(R):
            lo, hi = max(bounds[r], start), min(bounds[r + 1], start + t)
            if lo < hi:
                pieces.append((r, u, lo - start, hi - lo))
        start += t
    return T, bounds, pieces


def test_schedule_slots_unique_and_cover():
    """Each piece writes workspace slot (range + unit): slots are distinct,
    stay below kv_ranges + units, and the pieces tile every unit once in
    range order (what the combine walks)."""
    import random
    rnd = random.Random(0)
    for trial in range(200):
        B = rnd.randint(1, 40)
        Hkv = rnd.choice([1, 2, 8])
        skv = [rnd.choice([0, 1, 127, 128, 129, rnd.randint(0, 9000)]) for _ in range(B)]
        R = rnd.randint(1, 300)
        T, bounds, pieces = _ranges_pieces(skv, Hkv, R)
        slots = [r + u for r, u, _, _ in pieces]
        assert len(set(slots)) == len(slots)
        assert all(0 <= s < R + B * Hkv for s in slots)
        per_unit = {}
        for r, u, off, n in pieces:
            per_unit.setdefault(u, []).append((r, off, n))
        for u, lst in per_unit.items():
            assert [x[0] for x in lst] == sorted(x[0] for x in lst)
            pos = 0
            for r, off, n in lst:
                assert off == pos
                pos += n
            assert pos == (skv[u // Hkv] + 127) // 128
            # the combine locates the ranges of a unit by this formula
            t_u = pos
            s_u = sum((L + 127) // 128 for L in skv[: u // Hkv]) * Hkv + (u % Hkv) * t_u
            Re = min(R, T)
            r_of = lambda x: ((x + 1) * Re + T - 1) // T - 1
            assert r_of(s_u) == lst[0][0] and r_of(s_u + t_u - 1) == lst[-1][0]
            # every range from the first to the last holds a piece of the unit
            assert [x[0] for x in lst] == list(range(lst[0][0], lst[-1][0] + 1))


def test_plan_extend_takes_decode_path(lib):
    """A few queries against a long cache run as decode with G * Sq columns."""
    for (Hq, Hkv, Sq, dk) in [(64, 8, 4, 128), (16, 1, 8, 512), (4, 4, 16, 128), (16, 2, 2, 512)]:
        pl = binding.plan(5, Hq, Hkv, Sq, 4096, dk, dk, num_sms=148)
        G = Hq // Hkv
        assert pl["path"] == 1 and pl["heads_per_cta"] == 16
        assert pl["head_blocks"] == -(-G * Sq // 16)
        n = pl["partials"] * G * Sq
        r256 = lambda x: (x + 255) // 256 * 256
        counters = 5 * Hkv * pl["head_blocks"]
        assert pl["workspace_bytes"] == r256(n * dk * 4) + r256(n * 4) + r256(counters * 4)
    for Sq in (3, 32, 100):  # not a power of two, or too many columns
        assert binding.plan(5, 64, 8, Sq, 4096, 128, 128, num_sms=148)["path"] == 0
    assert binding.plan(5, 128, 128, 4, 4096, 192, 128, num_sms=148)["path"] == 0


def test_plan_prefill(lib):
    # d = 512: SM pairs split the two matmuls (one CTA S and softmax, the
    # other O and PV); a work item is 128 query rows of one head, all of d_v
    pl = binding.plan(2, 16, 1, 4096, 4096, 512, 512, num_sms=148)
    assert pl["path"] == 0 and pl["dv_parts"] == 1 and pl["workspace_bytes"] == 0
    assert pl["grid_ctas"] == 148  # persistent: 74 pairs walk the 1024 work items
    pl = binding.plan(1, 3, 1, 129, 150, 512, 512, num_sms=148)
    assert pl["grid_ctas"] == 2 * 6  # 6 items (2 q tiles x 3 heads), one pair each
    pl = binding.plan(1, 64, 8, 8192, 8192, 128, 128, num_sms=148)
    assert pl["dv_parts"] == 1 and pl["grid_ctas"] == 148
    pl = binding.plan(1, 2, 1, 100, 100, 128, 128, num_sms=148)
    assert pl["grid_ctas"] == 2  # fewer work items than SMs
    # expanded MLA prefill: q/k 192 wide, v 128 wide, one d_v part
    pl = binding.plan(1, 128, 128, 4096, 4096, 192, 128, num_sms=148)
    assert pl["path"] == 0 and pl["dv_parts"] == 1 and pl["grid_ctas"] == 148


@pytest.mark.parametrize("args,code", [
    ((0, 16, 1, 1, 100, 512, 512), binding.ATTN_EINVAL),
    ((1, 16, 3, 1, 100, 512, 512), binding.ATTN_EINVAL),       # Hq % Hkv != 0
    ((1, 16, 1, 1, 0, 512, 512), binding.ATTN_EINVAL),         # no keys at all
    ((1, 16, 1, 1, 100, 256, 256), binding.ATTN_EUNSUPPORTED),
    ((1, 16, 1, 4, 100, 576, 512), binding.ATTN_EUNSUPPORTED),  # MLA shape is decode-only
    ((1, 16, 16, 1, 100, 192, 128), binding.ATTN_EUNSUPPORTED),  # expanded MLA: prefill only
    ((1, 16, 1, 1, 100, 512, 128), binding.ATTN_EUNSUPPORTED),
])
def test_plan_rejects(lib, args, code):
    pl = binding.Plan()
    assert lib.attn_plan(*args, 0, 148, ctypes.byref(pl)) == code
    assert binding.workspace_bytes(*args) == 0


def _call(lib, **over):
    """attn_fwd with fake but well-formed arguments; every case below must be
    rejected before any CUDA work, so the fake pointers are never used."""
    a = dict(q=0x10000, k=0x20000, v=0x30000, out=0x40000, lse=None, B=2, Hq=16, Hkv=1, Sq=1,
             skv=0x50000, max_skv=256, d_k=512, d_v=512, scale=0.04, causal=1, dtype=0,
             sq=binding.Strides(16 * 512, 512, 512), sk=binding.Strides(256 * 512, 256 * 512, 512),
             sv=binding.Strides(256 * 512, 256 * 512, 512), so=binding.Strides(16 * 512, 512, 512),
             ws=0x60000, ws_n=1 << 30, stream=None)
    a.update(over)
    return binding.fwd_raw(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["Hq"], a["Hkv"],
                           a["Sq"], a["skv"], a["max_skv"], a["d_k"], a["d_v"], a["scale"],
                           a["causal"], a["dtype"], a["sq"], a["sk"], a["sv"], a["so"], a["ws"],
                           a["ws_n"], a["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(q=None), binding.ATTN_EINVAL),
    (dict(skv=None), binding.ATTN_EINVAL),
    (dict(k=0x20008), binding.ATTN_EINVAL),                         # not 16-byte aligned
    (dict(sk=binding.Strides(256 * 512, 256 * 512, 516)), binding.ATTN_EINVAL),  # stride % 8
    (dict(sv=binding.Strides(-8, 0, 512)), binding.ATTN_EINVAL),
    (dict(causal=2), binding.ATTN_EINVAL),
    (dict(scale=float("nan")), binding.ATTN_EINVAL),
    (dict(scale=-0.5), binding.ATTN_EINVAL),
    (dict(scale=0.0), binding.ATTN_EINVAL),
    (dict(Hkv=3), binding.ATTN_EINVAL),
    (dict(dtype=7), binding.ATTN_EINVAL),
    (dict(d_k=64, d_v=64), binding.ATTN_EUNSUPPORTED),
    (dict(ws=None), binding.ATTN_EWORKSPACE),
    (dict(ws_n=64), binding.ATTN_EWORKSPACE),
    (dict(ws=0x60004), binding.ATTN_EWORKSPACE),
])
def test_fwd_rejects_before_launch(lib, over, code):
    assert _call(lib, **over) == code


@pytest.mark.parametrize("over,code", [
    (dict(q=None), binding.ATTN_EINVAL),
    (dict(idx=None), binding.ATTN_EINVAL),
    (dict(n_sel=None), binding.ATTN_EINVAL),
    (dict(n_sel=0x50002), binding.ATTN_EINVAL),          # int32 array not 4-byte aligned
    (dict(cache=0x20008), binding.ATTN_EINVAL),          # not 16-byte aligned
    (dict(idx_stride=100), binding.ATTN_EINVAL),         # rows shorter than topk
    (dict(topk=0), binding.ATTN_EINVAL),
    (dict(max_skv=0), binding.ATTN_EINVAL),
    (dict(sc=binding.Strides(256 * 576, 256 * 576, 0)), binding.ATTN_EINVAL),  # row stride 0
    (dict(scale=0.0), binding.ATTN_EINVAL),
    (dict(dtype=7), binding.ATTN_EINVAL),
    (dict(d_k=512, d_v=512), binding.ATTN_EUNSUPPORTED),  # the one-pass path is MLA only
    (dict(ws=None), binding.ATTN_EWORKSPACE),
    (dict(ws_n=64), binding.ATTN_EWORKSPACE),
])
def test_topk_fwd_rejects_before_launch(lib, over, code):
    """attn_topk_fwd validates its arguments before anything reaches the
    device (the fake pointers below are never dereferenced)."""
    a = dict(q=0x10000, cache=0x20000, out=0x40000, lse=None, B=2, Hq=128, idx=0x70000,
             idx_stride=256, n_sel=0x50000, skv=0x58000, topk=256, max_skv=4096, d_k=576,
             d_v=512, scale=0.07, dtype=0, sq=binding.Strides(128 * 576, 576, 576),
             sc=binding.Strides(4096 * 576, 4096 * 576, 576),
             so=binding.Strides(128 * 512, 512, 512), ws=0x60000, ws_n=1 << 30)
    a.update(over)
    assert binding.topk_raw(a["q"], a["cache"], a["out"], a["lse"], a["B"], a["Hq"], a["idx"],
                            a["idx_stride"], a["n_sel"], a["skv"], a["topk"], a["max_skv"],
                            a["d_k"], a["d_v"], a["scale"], a["dtype"], a["sq"], a["sc"], a["so"],
                            a["ws"], a["ws_n"], None) == code


@pytest.mark.parametrize("over,code", [
    (dict(kc=None), binding.ATTN_EINVAL),
    (dict(skv=None), binding.ATTN_EINVAL),
    (dict(dk=100), binding.ATTN_EINVAL),                 # not a multiple of 8 elements
    (dict(kn=0x20008), binding.ATTN_EINVAL),             # not 16-byte aligned
    (dict(vn=None), binding.ATTN_EINVAL),                # separate V cache needs v_new
    (dict(B=0), binding.ATTN_EINVAL),
    (dict(dtype=9), binding.ATTN_EINVAL),
])
def test_cache_append_rejects_before_launch(lib, over, code):
    """attn_cache_append validates its arguments before anything reaches the
    device (the fake pointers below are never dereferenced)."""
    a = dict(kc=0x10000, vc=0x30000, kn=0x20000, vn=0x40000, skv=0x50000, B=2, Hkv=1,
             max_skv=64, dk=128, dv=128, dtype=0)
    a.update(over)
    s = binding.Strides(64 * 128, 64 * 128, 128)
    sn = binding.Strides(128, 128, 128)
    assert lib.attn_cache_append(a["kc"], a["vc"], a["kn"], a["vn"], a["skv"], a["B"], a["Hkv"],
                                 a["max_skv"], a["dk"], a["dv"], a["dtype"], s, s, sn, sn,
                                 None) == code


@pytest.mark.parametrize("over,code", [
    (dict(src=None), binding.ATTN_EINVAL),
    (dict(idx=None), binding.ATTN_EINVAL),
    (dict(dst_len=None), binding.ATTN_EINVAL),
    (dict(idx=0x50002), binding.ATTN_EINVAL),            # int32 array not 4-byte aligned
    (dict(dst=0x20008), binding.ATTN_EINVAL),            # not 16-byte aligned
    (dict(d=100), binding.ATTN_EINVAL),                  # not a multiple of 8 elements
    (dict(topk=0), binding.ATTN_EINVAL),
    (dict(idx_stride=8), binding.ATTN_EINVAL),           # rows shorter than topk
    (dict(dtype=5), binding.ATTN_EINVAL),
    (dict(H=70000), binding.ATTN_EUNSUPPORTED),
])
def test_gather_rows_rejects_before_launch(lib, over, code):
    """attn_gather_rows validates its arguments before anything reaches the
    device (the fake pointers below are never dereferenced)."""
    a = dict(src=0x10000, dst=0x20000, idx=0x50000, n_sel=0x60000, skv=0x70000,
             dst_len=0x80000, B=2, H=1, topk=16, d=576, dtype=0, idx_stride=16)
    a.update(over)
    ss = binding.Strides(4096 * a["d"], 4096 * a["d"], a["d"])
    sd = binding.Strides(16 * a["d"], 16 * a["d"], a["d"])
    assert lib.attn_gather_rows(a["src"], a["dst"], a["idx"], a["n_sel"], a["skv"], a["dst_len"],
                                a["B"], a["H"], a["topk"], a["d"], a["dtype"], ss, sd,
                                a["idx_stride"], None) == code


def test_binding_rejects_host_tensors(lib):
    """A CPU tensor never reaches the library: its host address would be an
    illegal access in a kernel."""
    import torch

    q = torch.zeros(1, 16, 1, 512, dtype=torch.bfloat16)
    k = torch.zeros(1, 1, 64, 512, dtype=torch.bfloat16)
    out = torch.zeros(1, 16, 1, 512, dtype=torch.bfloat16)
    skv = torch.tensor([64], dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        binding.attn_fwd(q, k, k, out, skv, 64, 0.04)
    with pytest.raises(ValueError, match="CUDA"):
        binding.attn_fwd_noalloc(q, k, k, out, skv, 64, 0.04)
    with pytest.raises(ValueError, match="CUDA"):
        binding.cache_append(k, None, k[:, :, :1], None, skv)
    idx = torch.zeros(1, 8, dtype=torch.int32)
    dst = torch.zeros(1, 1, 8, 512, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        binding.gather_rows(k, dst, idx, skv, skv, torch.zeros(1, dtype=torch.int32))
