"""Host logic of bench.py that needs no GPU: naming the dominant kernel from a live profile."""
import bench


def _cat(launches, ms, flops=0.0, nbytes=0.0):
    return dict(launches=launches, total_ms=ms, flops=flops, bytes=nbytes)


def test_rank_kernels_takes_off_event_overhead_and_groups_launch_kinds():
    # per-step figures of an 8B SFT step (3 steps): many short LoRA launches would outrank the
    # NF4 GEMMs if the event pair's own cost per launch stayed in
    prof = {"h2d_layer_copy": _cat(180, 366.0), "gemm_nf4_fwd": _cat(384, 49.3, 1e13, 1e10),
            "gemm_nf4_dx": _cat(384, 49.2, 1e13, 1e10), "gemm_lora": _cat(1056, 53.1, 1e11, 1e10),
            "gemm_lora_grad": _cat(1056, 40.3, 1e11, 1e10), "rmsnorm": _cat(390, 11.0),
            "event_overhead": _cat(24, 0.144)}
    kern, grouped, dom, ov_ms = bench.rank_kernels(prof)
    assert abs(ov_ms - 0.006) < 1e-12
    assert "h2d_layer_copy" not in kern and "event_overhead" not in prof
    assert dom == "gemm_nf4_fwd,gemm_nf4_dx"
    assert grouped[dom] == ("gemm_nf4_fwd", "gemm_nf4_dx")
    assert abs(kern["gemm_lora"]["net_ms"] - (53.1 - 1056 * 0.006)) < 1e-9
    assert grouped["rmsnorm"] == ("rmsnorm",)


def test_rank_kernels_without_overhead_or_groups():
    kern, grouped, dom, ov_ms = bench.rank_kernels({"attention_fwd": _cat(32, 2.0), "rope": _cat(64, 1.0)})
    assert ov_ms == 0.0 and dom == "attention_fwd"
    assert bench.rank_kernels({"h2d_layer_copy": _cat(1, 1.0)})[2] is None


def test_both_arms_print_the_same_config():
    wl = bench.WORKLOADS[bench.DEFAULT]
    a = bench.config_of(bench.DEFAULT, wl, 1)
    assert a == bench.config_of(bench.DEFAULT, dict(wl), 1)
    assert a["global_batch"] == wl["B"] and a["seq_len"] == wl["S"] and a["parallelism"] == "dp1"
    assert bench.config_of(bench.DEFAULT, wl, 4)["global_batch"] == 4 * wl["B"]
