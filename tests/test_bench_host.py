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
    import json
    for kernel in ("flash", "qk_stats", "softmax_av"):
        digest = bench.source_digest(kernel)
        good = tmp_path / f"{kernel}.json"
        good.write_text(json.dumps({"source_digest": digest, "dram_bytes_read": 15799552, "dram_bytes_write": 0}))
        monkeypatch.setitem(bench.PROFILE_JSON, kernel, str(good))
        assert bench.profiled_traffic(kernel) == 15799552.0
        stale = tmp_path / f"{kernel}_stale.json"
        stale.write_text(json.dumps({"source_digest": "0123456789abcdef", "dram_bytes_read": 1,
                                     "dram_bytes_write": 0}))
        monkeypatch.setitem(bench.PROFILE_JSON, kernel, str(stale))
        assert bench.profiled_traffic(kernel) is None
        monkeypatch.setitem(bench.PROFILE_JSON, kernel, str(tmp_path / "missing.json"))
        assert bench.profiled_traffic(kernel) is None
    # each kernel's digest covers its own sources
    assert len({bench.source_digest(k) for k in ("flash", "qk_stats", "softmax_av")}) == 3


def test_both_arms_print_the_same_config():
    cfg = bench.job_config(1)
    assert cfg["flops_per_step"] == bench.STEP_FLOPS and cfg["calls_per_step"] == 32
    assert bench.SET_BYTES > 126e6          # each input set is larger than the L2
    assert bench.job_config(1) == cfg


def test_upload_groups_cover_the_calls_in_order():
    """The end-to-end leg's upload runs: consecutive, disjoint, covering every
    call once, at most the requested number, of about equal bytes."""
    sizes = [2 * c.B * c.H * (c.N + 2 * c.M) * c.d for c in synth.unet_step_set()]
    for groups in (1, 2, 4, 7, 32, 40):
        runs = bench.upload_groups(sizes, groups)
        assert runs[0][0] == 0 and runs[-1][1] == len(sizes)
        assert all(a < b for a, b in runs)
        assert all(runs[i][1] == runs[i + 1][0] for i in range(len(runs) - 1))
        assert len(runs) <= groups
    runs = bench.upload_groups(sizes, 4)
    per = [sum(sizes[a:b]) for a, b in runs]
    assert len(runs) == 4 and max(per) <= 1.25 * sum(sizes) / 4
    assert bench.upload_groups([10], 4) == [(0, 1)]
