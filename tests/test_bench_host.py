"""Host-side helpers of bench.py, on the CPU: the recorded DRAM traffic is reported only while the
kernel sources hash to the value its ncu summary was taken on, and the CPU baseline's sampler
cycles over the batch until its time budget is spent."""
import shutil

import bench
import workloads


def _profile(dirpath, kind, workload, source_hash, dram_bytes):
    f = dirpath / f"{kind}_{workload}.md"
    f.write_text(f"# summary\n\n- kernel_source_hash: {source_hash}\n"
                 f"- dram_bytes_per_launch: {dram_bytes}\n- algorithmic_bytes_per_launch: 1\n")
    return f


def test_recorded_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "PROFILE_DIR", tmp_path)
    h = bench.kernel_hash()
    _profile(tmp_path, "decode_kernel", "wl_a", h, 306134784)
    _profile(tmp_path, "decode_kernel", "wl_b", "0" * 16, 5)
    assert bench.recorded_traffic("wl_a") == 306134784
    assert bench.recorded_traffic("wl_b") is None          # taken on other sources
    assert bench.recorded_traffic("wl_missing") is None    # no summary
    hp = bench.kernel_hash(bench.PROJECT_SOURCES)
    _profile(tmp_path, "project_kernel", "wl_a", hp, 9466368)
    assert bench.recorded_traffic("wl_a", "project_kernel", bench.PROJECT_SOURCES) == 9466368
    assert bench.recorded_traffic("wl_a", "project_kernel") is None  # the attention kernel's hash


def test_kernel_hash_changes_with_any_source_byte(tmp_path, monkeypatch):
    csrc = tmp_path / "latent_kv_cache_mlra_b200" / "csrc"
    shutil.copytree(bench.ROOT / "latent_kv_cache_mlra_b200" / "csrc", csrc)
    monkeypatch.setattr(bench, "ROOT", tmp_path)
    before = bench.kernel_hash()
    f = csrc / bench.KERNEL_SOURCES[0]
    f.write_bytes(f.read_bytes() + b"\n")
    assert bench.kernel_hash() != before
    assert bench.kernel_hash(bench.PROJECT_SOURCES) == bench.kernel_hash(bench.PROJECT_SOURCES)


def test_cpu_baseline_sampler_cycles_over_the_batch():
    inp = workloads.make_inputs(workloads.get("tiny_mlra4_f32"))
    dt, done, threads = bench.time_oracle(inp, budget_s=0.3)
    assert done > inp.workload.batch and dt >= 0.3 and threads >= 1
