"""CPU checks of the bench's bookkeeping: the tile and FLOP counts that turn
kernel time into TFLOP/s (against brute force over the (query, key) pairs),
and the JSON line of the CPU-oracle arm (`--impl reference`)."""
import io
import os
import json
import types
from contextlib import redirect_stdout

import numpy as np
import pytest

import bench
from rope_context_extension_jet_b200 import inputs as I


def brute_tiles(L, w0, P=0, bm=128, bn=128):
    """Causal tiles and tiles holding both local (i - j < w0) and remote causal
    pairs, by listing every pair of every tile of query rows [P, L)."""
    tiles = band = 0
    for i0 in range(P, L, bm):
        i = np.arange(i0, min(i0 + bm, L))
        for j0 in range(0, int(i[-1]) + 1, bn):
            j = np.arange(j0, j0 + bn)
            diff = i[:, None] - j[None, :]
            causal = (diff >= 0) & (j[None, :] < L)
            if not causal.any():
                continue
            tiles += 1
            local = causal & (diff < w0)
            if local.any() and (causal & ~local).any():
                band += 1
    return tiles, band


@pytest.mark.parametrize("L,w0,P", [(700, 200, 0), (1000, 1, 0), (1000, 0, 0), (513, 513, 0),
                                    (1300, 300, 640), (1300, 129, 1200), (257, 128, 0)])
def test_tile_counts_match_brute_force(L, w0, P):
    assert bench.tile_counts(L, w0, P=P) == brute_tiles(L, w0, P=P)


def test_headline_tile_counts():
    # 128K, w0 = 4096, 128 x 128 tiles: 1024 query blocks, 524,800 causal tiles,
    # the band i - j = 4096 crossing 992 of them
    assert bench.tile_counts(131072, 4096) == (524800, 992)


def test_prefill_flops_against_row_sums():
    w = I.PrefillWorkload("t", 1, "bf16", 2, 4, 2, 64, 1300, 500, 300, 1e4)
    for P in (0, 640):
        useful, computed, tiles, band = bench.prefill_flops(w, P=P)
        rows = np.arange(P, w.L, dtype=np.float64)
        # QK^T and P.V: 2 * d FLOPs each per causal (i, j) pair, j in [0, i]
        assert useful == pytest.approx(float(np.sum(4.0 * w.d * (rows + 1))) * w.Hq * w.B, rel=1e-12)
        # every causal tile computes a full 128 x 128 QK^T and P.V, band tiles one more QK^T
        assert computed == w.B * w.Hq * (tiles * 4.0 + band * 2.0) * w.d * 128 * 128
        assert computed >= useful


def test_reference_arm_json_line(monkeypatch):
    real = bench.oracle_prefill_sample
    monkeypatch.setattr(bench, "oracle_prefill_sample",
                        lambda w, budget_s, **kw: real(w, budget_s=0.3, **kw))
    args = types.SimpleNamespace(gpus=1, steps=1, warmup=3)
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(args, 0, 1)
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"):
        assert key in line, key
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["value"] > 0 and line["unit"] == "TFLOP/s" and line["higher_is_better"] is True
    assert line["config"]["workload"] == I.C4.name and line["config"]["G"] == 4
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_print_nothing():
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(types.SimpleNamespace(gpus=2, steps=1, warmup=3), 1, 2)
    assert buf.getvalue() == ""


def test_per_clock_figures():
    # 900.8 TFLOP/s at an 1852 MHz SM clock: 486.4 TFLOP/s per GHz, and 40.1% of
    # the tensor pipe's 148 SMs x 8192 FLOP/cycle at that clock
    peaks = {"bf16_tflops_sustained": 1401.4, "bf16_sustained_sm_mhz": 1335.0}
    r = bench.per_clock(900.8, 1852.0, peaks)
    assert r["tflops_per_ghz"] == pytest.approx(486.39, abs=0.01)
    assert r["frac_of_tensor_pipe_at_this_clock"] == pytest.approx(900.8e12 / (148 * 8192 * 1852e6), abs=1e-4)
    assert r["sustained_peak_tflops_per_ghz"] == pytest.approx(1401.4 / 1.335, abs=0.01)
    assert r["frac_of_sustained_peak_per_clock"] == pytest.approx(486.39 / (1401.4 / 1.335), abs=1e-3)
    assert bench.per_clock(900.8, None, peaks) is None


def test_peak_clock_lookup_searches_nested_keys():
    d = {"hbm_gbs": 6548.5, "bf16": {"sustained": {"sm_mhz_median_sustained": 1335}, "burst_sm_mhz": 1900},
         "mem_clock_mhz_sustained": 3996}
    assert bench._find_mhz(d, "sustain") == 1335.0


NCU_CSV = '''==PROF== Connected to process 4242
"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size","Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"
"0","4242","python3","127.0.0.1","prefill_pair_kernel(CUtensorMap_st, CUtensorMap_st, CUtensorMap_st, jl::tc::TcParams)","1","7","(512, 1, 1)","(2048, 8, 1)","0","10.0","Command line profiler metrics","gpu__time_duration.sum","ns","156,000,000"
"1","4242","python3","127.0.0.1","void jl::decode_tc_kernel<128, 4>(CUtensorMap_st, CUtensorMap_st, jl::DecodeProblem, jl::DecodeLaunch)","1","7","(160, 1, 1)","(4, 8, 8)","0","10.0","Command line profiler metrics","gpu__time_duration.sum","ns","800000"
"2","4242","python3","127.0.0.1","void jl::decode_tc_kernel<128, 4>(CUtensorMap_st, CUtensorMap_st, jl::DecodeProblem, jl::DecodeLaunch)","1","7","(160, 1, 1)","(4, 8, 8)","0","10.0","Command line profiler metrics","gpu__time_duration.sum","ns","1200000"
"2","4242","python3","127.0.0.1","void jl::decode_tc_kernel<128, 4>(CUtensorMap_st, CUtensorMap_st, jl::DecodeProblem, jl::DecodeLaunch)","1","7","(160, 1, 1)","(4, 8, 8)","0","10.0","Command line profiler metrics","dram__bytes_read.sum","byte","4,294,967,296"
==PROF== Disconnected from process 4242
'''


def test_ncu_csv_parsing_and_launch_shares():
    rows = bench.parse_ncu_csv(NCU_CSV)
    assert len(rows) == 4
    assert rows[0]["value"] == 156e6 and rows[3]["value"] == 4294967296.0
    summ = bench.launch_summary(rows)
    assert [s[0] for s in summ] == ["prefill_pair_kernel", "void jl::decode_tc_kernel<128, 4>"]
    (k0, n0, t0, s0), (k1, n1, t1, s1) = summ
    assert (n0, n1) == (1, 2)
    assert t0 == pytest.approx(156.0) and t1 == pytest.approx(2.0)
    assert s0 == pytest.approx(156.0 / 158.0) and s0 + s1 == pytest.approx(1.0)


def test_ncu_raw_csv_parsing():
    text = ('==PROF== noise\n"ID","Kernel Name","gpu__time_duration.sum","dram__bytes_read.sum"\n'
            '"","","ns","byte"\n"0","prefill_pair_kernel(...)","8,708,000","404,577,000"\n')
    rows = bench.parse_ncu_raw_csv(text)
    m = {r["metric"]: r["value"] for r in rows}
    assert m["gpu__time_duration.sum"] == 8708000.0 and m["dram__bytes_read.sum"] == 404577000.0
    assert rows[0]["kernel"].startswith("prefill_pair_kernel")


def test_ncu_all_regenerates_every_committed_profile():
    # one command (bench.py --ncu all) makes every summary profiles/ holds
    made = {bench.ncu_summary_name(mode, L) for mode, L in bench.NCU_ALL}
    prof = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "profiles")
    for f in os.listdir(prof):
        stem, ext = os.path.splitext(f)
        if ext in (".md", ".json") and stem != "traffic":
            assert stem in made, f"profiles/{f} is not made by bench.py --ncu all"
