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
