"""Host-side pieces of bench.py and the input generators (no GPU): the
source fingerprint that gates recorded DRAM traffic, the top-k accounting,
and the top-k selection generator."""
import json
import os

import torch

import bench
from attention_mqa_gqa_b200 import workloads as wl


def test_code_tokens_drops_comments_keeps_literals():
    src = ('int a = 1; // note\n/* block\n comment */ const char* s = "x // y /* z */";\n'
           "char q = '\"';   int   b;  // it's\n")
    assert bench.code_tokens(src) == 'int a = 1; const char* s = "x // y /* z */"; char q = \'"\'; int b;'
    # re-wrapping or rewording a comment leaves the fingerprint unchanged; code does not
    assert bench.code_tokens("x = 1; // one\n") == bench.code_tokens("x  =  1;\n// two\n")
    assert bench.code_tokens("x = 1;") != bench.code_tokens("x = 2;")


def test_recorded_traffic_matches_current_sources():
    """Every committed ncu traffic figure was taken on the kernel code as it
    is now (else bench.py reports traffic null)."""
    with open(os.path.join(bench.ROOT, "profiles", "ncu_traffic.json")) as f:
        d = json.load(f)
    for key, e in d.items():
        kernel, workload = key.split(":")
        assert e["sources_sha"] == bench.sources_hash(kernel), key
        assert bench.traffic_for(kernel, workload) == e["dram_bytes_per_launch"]


def test_make_selection():
    g = torch.Generator().manual_seed(0)
    skv = [5000, 100, 0, 2048]
    idx, n_sel = wl.make_selection(skv, 2048, g)
    assert n_sel.tolist() == [2048, 100, 0, 2048]
    for b, L in enumerate(skv):
        sel = idx[b, : n_sel[b]]
        assert len(set(sel.tolist())) == len(sel)              # distinct
        assert bool((sel[1:] > sel[:-1]).all())                 # ascending
        assert len(sel) == 0 or (0 <= int(sel.min()) and int(sel.max()) < L)
    assert sorted(idx[3].tolist()) == list(range(2048))         # skv == topk: every position


def test_topk_accounting():
    """A top-k step reads the selected rows once: kv bytes = selected rows x
    1152 B for the 576-wide latent rows."""
    w = wl.WORKLOADS["mla_topk_decode"].scaled(B=3, skv_lo=100, skv_hi=3000)
    inp = {"skv": torch.tensor([3000, 100, 2500], dtype=torch.int32),
           "n_sel": torch.tensor([2048, 100, 2048], dtype=torch.int32)}
    assert w.is_decode
    assert bench.keys_of(w, inp).tolist() == [2048, 100, 2048]
    assert bench.kv_bytes(w, bench.keys_of(w, inp)) == (2048 + 100 + 2048) * 576 * 2


def test_reference_arm_topk(monkeypatch, capsys):
    """`bench.py --impl reference` on a top-k workload: the numpy top-k oracle
    timed on the host, counted by the selected rows (a small instance of the
    mla_topk_decode recipe)."""
    import types

    small = wl.WORKLOADS["mla_topk_decode"].scaled(name="topk_small", B=2, Hq=16, skv_lo=300,
                                                   skv_hi=700, topk=128)
    monkeypatch.setitem(wl.WORKLOADS, "topk_small", small)
    args = types.SimpleNamespace(workload="topk_small", steps=1, warmup=0, ref_step_budget=0.5,
                                 gpus=1)
    assert bench.reference_arm(args, 1, 0) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["config"]["topk"] == 128 and "top-k" in line["cpu_baseline"]["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    # the reference arm names the same workload as the GPU arm: where each
    # runs is reported outside `config`
    inp = wl.make_inputs(small)
    assert line["config"] == bench.config_of(small, inp)
    assert "parallelism" not in line["config"] and line["parallelism"].startswith("host cores")


def test_timed_steps_give_many_replays():
    """20 timed steps are replayed as 10 graphs of two steps (K odd: one step
    per graph), so the step-time percentiles rest on many samples."""
    for k in (20, 100, 2):
        assert bench.steps_per_graph(k) == 2 and k // bench.steps_per_graph(k) == k // 2
    assert bench.steps_per_graph(21) == 1


def test_roofline_reports_measured_and_nominal_fractions():
    w = wl.WORKLOADS["mqa_decode"]
    skv = [1000, 3000]
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1300.0}
    ms = bench.kv_bytes(w, skv) / 4.0e12 * 1e3  # 4 TB/s
    r = bench.roofline(w, skv, ms, peaks, "measured", False, None)
    assert abs(r["frac"] - 4000 / 6000) < 1e-3 and abs(r["frac_nominal"] - 0.5) < 1e-3
    assert r["peak_nominal"] == 8000.0 and r["bound"] == "hbm"
    wp = wl.WORKLOADS["mqa_prefill"]
    ms = bench.flops(wp, [4096, 4096]) / 1.125e15 * 1e3  # 1125 TFLOP/s
    r = bench.roofline(wp, [4096, 4096], ms, peaks, "measured", True, None)
    assert abs(r["frac"] - 1125 / 1300) < 1e-3 and abs(r["frac_nominal"] - 0.5) < 1e-3


def test_clock_sampler_summary(tmp_path):
    """The clocks summary in the bench line: median SM MHz under load, the
    maximum, and every throttle reason seen active (parsed from the
    nvidia-smi CSV the sampler records; the sample file is removed)."""
    cs = bench.ClockSampler.__new__(bench.ClockSampler)
    cs.path = str(tmp_path / "clocks.csv")
    with open(cs.path, "w") as f:
        f.write("0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active\n")
        f.write("0, 1900, 1965, 900.1, 0x4, Not Active, Not Active, Not Active, Active\n")
        f.write("0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active\n")

    class _Proc:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            pass

    cs.proc, cs.f = _Proc(), open(os.devnull, "w")
    assert cs.stop() == {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                         "samples": 3}
    assert not os.path.exists(cs.path)


def test_dominant_kernel_names():
    """The roofline names the kernel each path runs (d = 512 prefill: the
    split-matmul pairs), and every named kernel has its sources listed, so a
    recorded traffic figure can be matched to the code it was taken on."""

    class G:
        def __init__(self, decode):
            self.decode = decode

    names = set()
    for name, w in wl.WORKLOADS.items():
        k = bench.kernel_name(w, G(w.is_decode))
        names.add(k)
        if not w.is_decode:
            assert k == ("prefill_ab_kernel" if w.d_k == 512 else "prefill_kernel"), name
        elif w.mla:
            assert k == "mla_pair_kernel", name
        else:
            assert k == "decode_split_kernel", name
    assert names <= set(bench.KERNEL_SOURCES)
    for srcs in bench.KERNEL_SOURCES.values():
        for f in srcs:
            assert os.path.exists(os.path.join(bench.ROOT, f)), f
