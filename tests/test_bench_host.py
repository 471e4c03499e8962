"""Host-side logic of bench.py (CPU only): the DRAM traffic figures it reports come from the ncu
summaries in profiles/ only while the kernel's source is the one those counters were taken on."""
import os

import bench


def test_stale_or_missing_profile_gives_no_traffic(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    digest = bench.source_digest(bench.GEMM_SOURCES)
    (prof / "fresh.txt").write_text(f"x\ntraffic_bytes_per_launch: 1.5e7 source: {digest}\n")
    (prof / "stale.txt").write_text("traffic_bytes_per_launch: 1.5e7 source: 0123456789abcdef\n")
    (prof / "none.txt").write_text("no traffic line here\n")
    real_root = bench.ROOT
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # the digest still reads the kernel sources of the repository
    monkeypatch.setattr(bench, "source_digest",
                        lambda names=bench.ATTN_SOURCES: digest if names == bench.GEMM_SOURCES
                        else "ffffffffffffffff")
    assert bench.profile_traffic("fresh.txt", bench.GEMM_SOURCES) == 1.5e7
    assert bench.profile_traffic("stale.txt", bench.GEMM_SOURCES) is None
    assert bench.profile_traffic("none.txt", bench.GEMM_SOURCES) is None
    assert bench.profile_traffic("missing.txt", bench.GEMM_SOURCES) is None
    assert bench.profile_traffic("fresh.txt", bench.CONV_SOURCES) is None
    assert os.path.isdir(real_root)


def test_source_digest_tracks_the_kernel_files():
    a = bench.source_digest(bench.ATTN_SOURCES)
    assert a == bench.kernel_source_digest()
    assert len({a, bench.source_digest(bench.GEMM_SOURCES), bench.source_digest(bench.CONV_SOURCES)}) == 3


def _args(**kw):
    import argparse
    d = dict(q_rope="append", scaling="weak", workload="wan_full")
    d.update(kw)
    return argparse.Namespace(**d)


def test_both_arms_print_the_same_config():
    """The reference arm (the oracle on the host) describes the workload with the very object
    the CUDA arm prints, so the two lines are comparable key by key."""
    from causal_video_diffusion_b200 import workloads as W
    wl = W.WORKLOADS["wan_full"]
    for world in (1, 2, 8):
        for scaling in ("weak", "strong"):
            a = bench.arm_config(wl, world, _args(scaling=scaling))
            b = bench.arm_config(wl, world, _args(scaling=scaling))
            assert a == b
            assert a["workload"].startswith("wan_full: B=1 H=12 D=128")
    assert "shards x8" in bench.arm_config(wl, 8, _args(scaling="strong"))["parallelism"]
    assert "independent" in bench.arm_config(wl, 8, _args())["parallelism"]


def test_gpus_flag_starts_its_own_ranks(monkeypatch):
    """``bench.py --gpus N`` with no launcher environment runs itself as N ranks on 127.0.0.1."""
    calls = []
    monkeypatch.setattr(bench.subprocess, "call", lambda cmd: calls.append(cmd) or 0)
    assert bench.launch_ranks(4, ["--gpus", "4", "--steps", "3"], port=29512) == 0
    cmd = calls[0]
    i = cmd.index("-m")
    assert cmd[i + 1] == "torch.distributed.run"
    assert "--nproc-per-node=4" in cmd and "--nnodes=1" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[cmd.index("--master-port") + 1] == "29512"
    assert cmd[0] == "timeout" and cmd[-3:] == ["--gpus", "4", "--steps", "3"][-3:]
    assert cmd[-5].endswith("bench.py")


def test_clock_summary_keeps_only_the_timed_region():
    """Samples taken before or after the timed region (an idle GPU at its maximum clock) do not
    enter the summary; a region shorter than the sampling interval is stood for by the nearest
    sample, and the line says so."""
    import datetime
    base = datetime.datetime(2026, 12, 3, 3, 0, 0)

    def row(dt_ms, mhz, cap):
        ts = (base + datetime.timedelta(milliseconds=dt_ms)).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        flags = "Active" if cap else "Not Active"
        return f"{ts}, 0, {mhz}, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, {flags}\n"

    lines = [row(0, 1965, False), row(50, 1965, False), row(300, 1770, True), row(350, 1755, True),
             row(400, 1785, True), row(700, 1965, False), "garbage line\n"]
    t = base.timestamp()
    s = bench.summarize_clocks(lines, t + 0.29, t + 0.41)
    assert s["samples"] == 3 and s["sm_mhz"] == 1770 and s["reasons"] == ["sw_power_cap"]
    assert s["window"] == "timed region"
    s = bench.summarize_clocks(lines, t + 0.51, t + 0.52)  # between samples: the nearest one
    assert s["samples"] == 1 and s["window"].startswith("nearest") and s["sm_mhz"] == 1785
    assert bench.summarize_clocks(["x\n"], t, t)["reasons"] == ["unsampled"]


def test_other_workloads_summary_on_stub_legs(monkeypatch):
    """The default line's summary of the other workloads: one entry per leg with its headline
    fields, the clip run with its own step count, and a failing leg recorded as an error instead
    of losing the line."""
    import argparse
    seen = {}

    def fake(kind):
        def run(a, rank, local_rank, world, emit=True):
            assert emit is False and world == 1 and a.no_cpu_baseline and a.no_other_workloads
            seen[a.workload] = (a.steps, a.warmup)
            if a.workload == "vae_conv":
                raise RuntimeError("device error in the convolution")
            r = {"config": {"workload": a.workload + ": shape"}, "value": 1.0, "unit": "TFLOP/s",
                 "ms_per_step": 2.0, "steps": a.steps,
                 "roofline": {"frac": 0.5, "kernel": kind, "traffic": None},
                 "clocks": {"sm_mhz": 1965.0, "reasons": [], "samples": 2}}
            if kind == "attn":
                r["rope_roofline"] = {"achieved": 5000.0, "frac": 0.76}
                r["chunk_steps_per_s"] = 1234.0
            return r
        return run

    monkeypatch.setattr(bench, "run_ours", fake("attn"))
    monkeypatch.setattr(bench, "run_lowrank", fake("gemm"))
    monkeypatch.setattr(bench, "run_vae_conv", fake("conv"))
    monkeypatch.setattr(bench, "run_clip", fake("clip"))
    args = argparse.Namespace(workload="wan_full", steps=400, warmup=10, no_cpu_baseline=False,
                              no_other_workloads=False, seed=1, q_rope="append", scaling="weak")
    out = bench.other_workloads(args, 0)
    assert list(out) == list(bench.OTHER_WORKLOADS)
    assert seen["wan_window"] == (20, 5) and seen["clip30"] == (3, 3)
    assert out["wan_window"]["rope_frac"] == 0.76 and out["wan_window"]["roofline_frac"] == 0.5
    assert out["lowrank_vo"]["roofline_kernel"] == "gemm" and "rope_frac" not in out["lowrank_vo"]
    assert out["vae_conv"] == {"error": "RuntimeError: device error in the convolution"}
    assert args.workload == "wan_full" and args.steps == 400   # the caller's args untouched
