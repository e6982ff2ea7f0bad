"""Host-side arithmetic of bench.py (no GPU needed): the op count behind the
effective TOP/s, the whole-job throughput, the roofline peaks, the L2 note of
the timing rule, and the source keys of the committed DRAM traffic."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_ops_per_image_block_counts_the_method_macs():
    # ViT-B, 197 tokens: 24 N D^2 + 4 N^2 D integer ops (2 x MAC)
    N, D = 197, 768
    assert bench.ops_per_image_block(N, D) == 2 * (12 * N * D * D + 2 * N * N * D)
    # the block total of the ViT-B b64 workload: 186 G ops
    assert abs(64 * bench.ops_per_image_block(N, D) / 1e9 - 186.1) < 0.1


def test_whole_job_throughput():
    # 4 ranks x 64 images x 100 steps in 2 s of the slowest rank
    assert bench.whole_job_images_per_s(4, 64, 100, 2000.0) == pytest.approx(12800.0)
    assert bench.whole_job_images_per_s(1, 64, 10, 1.6) == pytest.approx(400000.0)


def test_peaks_for_each_bound():
    peaks = {"hbm_gbs": 6459.3, "bf16_tflops": 1679.9, "bf16_tflops_sustained": 1419.0, "sm_max_mhz": 1965.0}
    pk, unit, _ = bench.peak_for("tensor", peaks, 148)
    assert unit == "TOP/s" and pk == pytest.approx(2 * 1679.9)
    pk, unit, _ = bench.peak_for("alu", peaks, 148)
    assert unit == "TOP/s" and pk == pytest.approx(148 * 128 * 1965e6 / 1e12)
    pk, unit, _ = bench.peak_for("hbm", peaks, 148)
    assert unit == "GB/s" and pk == pytest.approx(6459.3)


def test_l2_note_says_whether_inputs_exceed_l2():
    l2 = 126 * 2 ** 20
    big = bench.l2_note(28, 64 * 197 * 768, l2)
    assert ">" in big and "L2" in big
    small = bench.l2_note(64, 197 * 192, l2)
    assert ">" not in small and "L2-resident" in small


def test_every_timed_kernel_has_a_source_key():
    names = ["layernorm", "gemm_qkv", "gemm_qkv_round_half_up", "attention", "attention_logits16",
             "gemm_o_residual", "gemm_fc1_shiftgelu", "gemm_fc2_residual", "shiftgelu_standalone"]
    for n in names:
        files = bench.kernel_sources(n, os.path.join(ROOT, "integer_only_quantized_int8_b200", "csrc"),
                                     os.path.join(ROOT, "include"))
        assert all(os.path.exists(f) for f in files), n
        assert len(bench.kernel_source_hash(n)) == 16


def test_traffic_entries_follow_their_kernels_sources():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        tab = json.load(f)
    for key, ent in tab.items():
        kernel, workload = key.split("@")
        got = bench.load_traffic(kernel, workload)
        if ent["source_hash"] == bench.kernel_source_hash(kernel):
            assert got == float(ent["dram_bytes_per_launch"]), key
        else:
            assert got is None, key
    assert bench.load_traffic("attention", "no_such_workload") is None


def test_gpu_local_cpus_is_a_subset_of_the_allowed_cpus_or_none():
    # on a host without a GPU (or without NVML) the end-to-end buffers keep
    # the process's own affinity
    cpus = bench.gpu_local_cpus(0)
    assert cpus is None or (cpus and cpus <= os.sched_getaffinity(0))


def test_profile_op_flag_parses():
    old = sys.argv
    try:
        sys.argv = ["bench.py", "--profile-op", "gemm_o_residual", "--kernel-reps", "2"]
        args = bench.parse_args()
    finally:
        sys.argv = old
    assert args.profile_op == "gemm_o_residual" and args.kernel_reps == 2
