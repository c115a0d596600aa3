"""bench.py's host logic, without a GPU: the roofline denominators come from
the measured peaks, whole-job throughput is bytes over the slowest rank's
time, the end-to-end leg's staging buffer holds every per-step input at a
256-byte boundary (one host-to-device copy per step), and the committed
DRAM-traffic summary is only used for the kernel source it was taken on."""
import json

import pytest
import torch

import synth


def test_peaks_are_the_measured_ones(tmp_path, monkeypatch):
    import bench
    # the measured copy bandwidth and bf16 GEMM burst figure when the peaks
    # file is present ...
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm_gbs": 6527.8, "bf16_tflops": 1642.8, "bf16_tflops_sustained": 1384.4}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.peaks() == (6527.8, 1642.8, "measured")
    # ... else the earlier measurement on this hardware, labelled as a fallback
    (tmp_path / "MEASURED_PEAKS.json").unlink()
    assert bench.peaks() == (6650.0, 1590.0, "fallback")


def test_job_throughput_is_all_ranks_bytes_over_the_slowest_time():
    import bench
    # 2 ranks x 3 steps x 1 GB in 0.5 s -> 12 GB/s
    assert bench.job_throughput(10**9, 2, 3, 500.0) == pytest.approx(12.0)
    assert bench.max_over_ranks(7.5, 1) == 7.5


def test_staging_buffer_layout(monkeypatch):
    import bench
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)  # no GPU here
    w = synth.llama3_8b_gqa_decode(num_seqs=16)
    st = bench.DecodeStep(w, torch.device("cpu"))
    base = st.d_stage.data_ptr()
    views = [st.q, st.nk, st.nv, st.bt, st.ctx, st.lens]
    wants = [w.query, w.new_key, w.new_value, w.block_tables, w.context_lens,
             (w.context_lens + 1).to(torch.int32)]
    end = 0
    for v, want in zip(views, wants):
        assert torch.equal(v, want)
        off = v.data_ptr() - base
        assert off % 256 == 0 and off >= end  # aligned, in order, no overlap
        end = off + v.numel() * v.element_size()
    assert st.h2d_bytes == st.h_stage.numel() >= end
    assert st.d2h_bytes == st.out.numel() * st.out.element_size()
    assert st.launches_per_step == 2  # decode with the fused append, split-KV combine


def test_traffic_is_reported_only_for_the_profiled_kernel_source(tmp_path, monkeypatch):
    import bench
    prof = tmp_path / "decode.md"
    prof.write_text("dram_bytes_per_algorithmic_byte: 1.25000\n"
                    f"kernel_source_sha256_16: {bench.kernel_hash()}\n")
    monkeypatch.setattr(bench, "PROFILE", str(prof))
    assert bench.profiled_traffic(1000.0) == pytest.approx(1250.0)
    prof.write_text("dram_bytes_per_algorithmic_byte: 1.25000\n"
                    "kernel_source_sha256_16: 0000000000000000\n")
    assert bench.profiled_traffic(1000.0) is None


def test_reference_arm_prints_the_contract_line(capsys, monkeypatch):
    import argparse

    import bench
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    assert bench.run_reference(argparse.Namespace(steps=2, warmup=3)) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["metric"] == bench.METRIC and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
