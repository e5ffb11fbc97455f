"""Host-side logic of bench.py that needs no GPU: the step set it times, the
form each call takes, the whole-job throughput, and the gate that reports the
flash kernel's DRAM traffic only while the profiled sources are unchanged."""
import bench
import synth


def test_step_set_is_the_unet_attention_set():
    assert len(bench.CALLS) == 32
    assert bench.STEP_FLOPS == sum(4 * c.B * c.H * c.N * c.M * c.d for c in bench.CALLS)
    # the 64x64 self-attention calls carry most of the work and are the ones the roofline times
    dom = [c for c in bench.CALLS if bench.is_dominant(c)]
    assert len(dom) == 5
    assert all(c.N == c.M == 4096 and c.d == 40 for c in dom)
    assert sum(c.flops for c in dom) == 5 * synth.WORKLOADS["self64"].flops


def test_policy_takes_flash_only_at_head_width_40():
    forms = {(c.d, bench.policy_form(c)) for c in bench.CALLS}
    assert forms == {(40, "flash"), (80, "partial"), (160, "partial")}


def test_job_throughput_counts_every_rank():
    one = bench.job_throughput(1, 10**12, 10, 1000.0)    # 10 steps of 1 TFLOP in 1 s
    assert abs(one - 10.0) < 1e-12
    assert abs(bench.job_throughput(4, 10**12, 10, 1000.0) - 4 * one) < 1e-12


def test_traffic_reported_only_for_the_profiled_source(tmp_path, monkeypatch):
    digest = bench.source_digest()
    good = tmp_path / "good.md"
    good.write_text(f"text\n\ntraffic_bytes_per_launch: 15799552 (source {digest})\n")
    monkeypatch.setattr(bench, "PROFILE_MD", str(good))
    assert bench.profiled_traffic() == 15799552.0
    stale = tmp_path / "stale.md"
    stale.write_text("traffic_bytes_per_launch: 15799552 (source 0123456789abcdef)\n")
    monkeypatch.setattr(bench, "PROFILE_MD", str(stale))
    assert bench.profiled_traffic() is None
    monkeypatch.setattr(bench, "PROFILE_MD", str(tmp_path / "missing.md"))
    assert bench.profiled_traffic() is None

