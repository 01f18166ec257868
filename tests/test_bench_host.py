"""Host-side pieces of bench.py: algorithmic byte counts, the source-hash
keyed DRAM traffic lookup and the clock-sample summary (no GPU)."""
import os
import sys
import time

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_alg_bytes_prefill_numbers():
    b = bench.alg_bytes(T=4096, T_real=4096, N_recv=25936, N_route=32768, H=7168, k=8, R=16,
                        idx_bytes=8)
    row = 7168 * 2
    assert b["dispatch_expand"] == 4096 * row + (25936 + 32768) * row + 4096 * 8 * 4 + 4096 * 16 * 4
    assert b["dispatch_expand"] == 900694016
    assert b["combine_reduce"] == 32768 * row + 4096 * row + 4096 * 8 * 8
    assert b["total"] == b["layout"] + b["dispatch_expand"] + b["combine_reduce"]


def test_alg_bytes_variants():
    two = bench.alg_bytes(128, 128, 833, 1024, 7168, 8, 16, 8, part_bytes=4)
    assert set(two) == {"layout", "dispatch_expand", "combine_local", "combine_epilogue", "total"}
    assert two["combine_local"] == 1024 * 14336 + 833 * 7168 * 4 + 128 * 8 * 8 + 128 * 16 * 4
    ne = bench.alg_bytes(128, 128, 833, 1024, 7168, 8, 16, 8, no_expand=True)
    assert "expand_index" in ne and ne["dispatch"] == 128 * 14336 + 833 * 14336 + 128 * 16 * 4


def test_alg_bytes_one_launch_step():
    """Layout and dispatch/expand as one kernel: the layout's bytes plus the
    copies, without the dispatch's re-read of pos / recv_pos."""
    sep = bench.alg_bytes(128, 128, 833, 1024, 7168, 8, 16, 8)
    one = bench.alg_bytes(128, 128, 833, 1024, 7168, 8, 16, 8, fused=True)
    assert set(one) == {"layout_dispatch_expand", "combine_reduce", "total"}
    assert one["layout_dispatch_expand"] == (sep["layout"] + sep["dispatch_expand"]
                                             - 128 * 8 * 4 - 128 * 16 * 4)
    assert one["combine_reduce"] == sep["combine_reduce"]


def test_step_call_choice_follows_the_library_threshold():
    from combine_ep_layout_07_b200 import epx
    a = bench.parse_args([])
    m = lambda T, k, argv=(): bench.step_mode(bench.parse_args(list(argv)), T, k)  # noqa: E731
    assert m(128, 8) == "one_launch" and m(128, 4) == "one_launch"
    assert m(4096, 8) == "paired"
    assert m(epx.FUSED_AUTO_MAX_ROUTES // 8, 8) == "one_launch"
    assert m(epx.FUSED_AUTO_MAX_ROUTES // 8 + 1, 8) == "paired"
    assert m(1, 16) == "one_launch" and m(1, 1) == "one_launch"
    assert m(0, 8) == "paired"          # empty batch: below the one-launch range
    assert m(128, 8, ["--step-calls", "separate"]) == "separate"
    assert m(960, 8, ["--step-calls", "fused"]) == "one_launch"
    assert m(4096, 8, ["--step-calls", "separate"]) == "separate"
    assert m(128, 8, ["--no-expand"]) == "separate"
    assert a.step_calls == "auto"


def test_alg_bytes_paired_step_keeps_the_position_reads():
    one = bench.alg_bytes(8, 1, 16, 16, 3584, 16, 32, 8, fused="one_launch")
    two = bench.alg_bytes(8, 1, 16, 16, 3584, 16, 32, 8, fused="paired")
    assert two["layout_dispatch_expand"] - one["layout_dispatch_expand"] == 8 * 16 * 4 + 8 * 32 * 4


def test_traffic_lookup_follows_source_and_engine(tmp_path, monkeypatch):
    h = bench.sources_hash("dispatch_expand")
    f = tmp_path / "traffic.txt"
    f.write_text("# comment\n"
                 f"kernel=dispatch_expand workload=prefill source={h} dram_bytes_per_launch=123 engine=bulk\n"
                 "kernel=dispatch_expand workload=decode source=0000 dram_bytes_per_launch=9 engine=vec\n")
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.committed_traffic("dispatch_expand", "prefill", "bulk") == 123.0
    assert bench.committed_traffic("dispatch_expand", "prefill", "vec") is None
    assert bench.committed_traffic("dispatch_expand", "decode", "vec") is None   # stale source
    assert bench.committed_traffic("no_such_kernel", "prefill") is None


def test_clock_summary_window_and_reasons(tmp_path):
    s = bench.ClockSampler("GPU-x")
    s.path = str(tmp_path / "clocks.csv")
    t0 = time.time()
    stamp = lambda t: time.strftime("%Y/%m/%d %H:%M:%S", time.localtime(t)) + ".000"  # noqa: E731
    lines = []
    for i, (mhz, pcap) in enumerate([(1965, "Not Active"), (1900, "Active"), (1965, "Not Active"),
                                     (1950, "Not Active")]):
        lines.append(f"{stamp(t0 + i)}, 0, {mhz}, 1965, 700.0, 0x0, Not Active, Not Active, "
                     f"Not Active, {pcap}")
    open(s.path, "w").write("\n".join(lines) + "\n")
    out = s.summary(t0 - 1, t0 + 5)
    assert out["samples"] == 4 and out["sm_max_mhz"] == 1965.0
    assert out["sm_mhz"] == pytest.approx(1957.5)
    assert out["reasons"] == ["sw_power_cap"] and out["window"] == "timed"


def test_default_arguments_fit_the_contract():
    a = bench.parse_args([])
    assert a.gpus == 1 and a.warmup >= 3 and a.steps > 0 and a.impl == "epx"
    assert a.workload == "prefill"


def test_step_stats_percentiles():
    # 1..101 ms: median 51, p10 11, p90 91 (nearest rank), reported in µs
    st = bench.step_stats([float(i) for i in range(101, 0, -1)])
    assert st == {"median": 51000.0, "p10": 11000.0, "p90": 91000.0}
    assert bench.step_stats([0.25]) == {"median": 250.0, "p10": 250.0, "p90": 250.0}


def test_host_cpu_reports_model_and_cores():
    h = bench.host_cpu()
    assert isinstance(h["model"], str)
    assert h["nproc"] == os.cpu_count()


def test_pinned_to_one_core_restores_affinity():
    before = os.sched_getaffinity(0)
    with bench.PinnedToOneCore() as pin:
        assert os.sched_getaffinity(0) == {pin.core}
    assert os.sched_getaffinity(0) == before


def test_split_pass_bytes_follow_the_step_options():
    """The split pass of separate calls (paired steps) is charged the same
    options as the step: two-stage partials, no-expand, index width."""
    tot = dict(T_real=4096, N_recv=25936, N_route=32768)
    for argv, part, keys in [([], None, {"layout", "dispatch_expand", "combine_reduce"}),
                             (["--two-stage", "fp32"], 4,
                              {"layout", "dispatch_expand", "combine_local", "combine_epilogue"}),
                             (["--no-expand"], None, {"layout", "dispatch", "expand_index",
                                                      "combine_reduce"})]:
        a = bench.parse_args(argv)
        sep = bench.step_alg_bytes(4096, tot, 7168, 8, 16, a, part, "separate")
        assert set(sep) - {"total"} == keys
        if not a.no_expand:
            pair = bench.step_alg_bytes(4096, tot, 7168, 8, 16, a, part, "paired")
            assert pair["total"] == sep["total"]
            assert pair["layout_dispatch_expand"] == sep["layout"] + sep["dispatch_expand"]
