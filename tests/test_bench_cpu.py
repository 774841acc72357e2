"""bench.py's roofline numerators and bookkeeping, on CPU.

The algorithmic bytes of each workload are the sums worked by hand in the
measurement table of the plan (packed words + s + z + x + y, fp16; never the
2 bytes per weight of a dense W), and the GEMM's FLOP are 2 M N K.
"""
import bench
import wq_inputs

# workload -> (packed words, s + z, x + y) bytes, worked by hand
HAND = {
    "tiny_gemv": (512 * 256 // 2, 2 * 2 * 4 * 256, 2 * 512 + 2 * 256),               # 71,168
    "decode_gemv_m1": (4096 * 4096 // 2, 2 * 2 * 32 * 4096, 2 * 4096 + 2 * 4096),    # 8,929,280
    "decode_gemv_m4": (4096 * 4096 // 2, 2 * 2 * 32 * 4096, 4 * (2 * 4096 + 2 * 4096)),
    "decode_gemv_m16": (4096 * 4096 // 2, 2 * 2 * 32 * 4096, 16 * (2 * 4096 + 2 * 4096)),
    "gemv_3bit": (11272192 + 5636096, 2 * 2 * 32 * 11008, 2 * 4096 + 2 * 11008),     # 18,347,520
    "sweep_1bit": (8192 * 8192 // 8, 2 * 2 * 64 * 8192, 4 * 8192),
    "sweep_2bit": (8192 * 8192 // 4, 2 * 2 * 64 * 8192, 4 * 8192),
    "sweep_8bit": (8192 * 8192, 2 * 2 * 64 * 8192, 4 * 8192),
    "sweep_8bit_perchannel": (8192 * 8192, 2 * 2 * 1 * 8192, 4 * 8192),
    "prefill_gemm": (4096 * 2048 // 2, 2 * 2 * 32 * 2048, 2 * 512 * 4096 + 2 * 512 * 2048),
}


def test_algorithmic_bytes_match_the_hand_sums():
    assert set(HAND) == set(wq_inputs.WORKLOADS)
    for name, parts in HAND.items():
        assert bench.algo_bytes(wq_inputs.WORKLOADS[name]) == sum(parts), name
    assert bench.algo_bytes(wq_inputs.WORKLOADS["decode_gemv_m1"]) == 8_929_280
    assert bench.algo_bytes(wq_inputs.WORKLOADS["tiny_gemv"]) == 71_168
    assert bench.algo_bytes(wq_inputs.WORKLOADS["gemv_3bit"]) == 18_347_520


def test_gemm_flops():
    assert bench.algo_flops(wq_inputs.WORKLOADS["prefill_gemm"]) == 8_589_934_592


def test_stack_exceeds_twice_the_l2():
    L2 = 126 * 2 ** 20
    for name, wl in wq_inputs.WORKLOADS.items():
        L = bench.layers_for(wl, L2)
        assert L * bench.algo_bytes(wl) > 2 * L2 or L == 1024, name


def test_traffic_lookup_needs_the_current_source(tmp_path, monkeypatch):
    """A capture counts only for the source digest it was taken on."""
    prof = tmp_path / "profiles"
    prof.mkdir()
    digest = bench.src_digest()
    (prof / "ncu_traffic.txt").write_text(
        "# header\n"
        f"kernel=k workload=w src={digest} dram_bytes_per_launch=123\n"
        "kernel=k workload=v src=000000000000 dram_bytes_per_launch=456\n")
    monkeypatch.setattr(bench, "ROOT", tmp_path)
    monkeypatch.setattr(bench, "src_digest", lambda: digest)
    assert bench.ncu_traffic("k", "w") == 123.0
    assert bench.ncu_traffic("k", "v") is None      # taken on another source
    assert bench.ncu_traffic("k", "x") is None
