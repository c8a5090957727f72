"""Host-side logic of bench.py: the workload arithmetic, the roofline selection, and the multi-rank
timing reduction (world size 2 over gloo on CPU)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def test_flop_counts():
    T, r = bench.TOKENS, bench.RANK_R
    main = sum(2 * T * N * K for N, K in bench.SHAPES)
    assert main == 2 * 8192 * (4096 * 4096 + 2 * 11008 * 4096)
    assert bench.step_flops() == 2 * main + sum(6 * T * r * (N + K) for N, K in bench.SHAPES)
    assert abs(bench.QUANT_B_PER_ELEM - 4.5159) < 1e-4 and abs(bench.DEQ_B_PER_ELEM - 2.5159) < 1e-4
    assert bench.step_flops() / 16 < bench.oracle_sample_flops() < bench.step_flops() / 10


def test_roofline_picks_the_dominant_class():
    prof = {"quantize": (3, 0.5), "dequantize": (3, 0.2), "fwd_gemm": (3, 3.0), "bwd_gemm": (3, 3.5), "lora": (30, 0.4)}
    peaks = {"hbm_gbs": 6543.1, "bf16_tflops": 1636.3, "bf16_tflops_sustained": 1375.0}
    rf = bench.roofline(prof, 1, peaks, "measured")
    assert rf["kernel"] == "bwd_gemm" and rf["bound"] == "tensor" and rf["peak"] == 1375.0
    flops = sum(2 * bench.TOKENS * N * K + 2 * bench.TOKENS * bench.RANK_R * K for N, K in bench.SHAPES)
    assert abs(rf["achieved"] - flops / 3.5e-3 / 1e12) < 0.01
    assert abs(rf["frac"] - rf["achieved"] / 1375.0) < 1e-3
    prof["quantize"] = (3, 9.0)
    assert bench.roofline(prof, 1, peaks, "measured")["bound"] == "hbm"


def test_roofline_peak_burst_for_a_short_region_at_full_clock():
    prof = {"quantize": (3, 0.5), "dequantize": (3, 0.2), "fwd_gemm": (3, 3.6), "bwd_gemm": (3, 3.5), "lora": (30, 0.4)}
    peaks = {"hbm_gbs": 6543.1, "bf16_tflops": 1636.3, "bf16_tflops_sustained": 1375.0}
    full = {"sm_mhz": 1965.0, "sm_max_mhz": 1965}
    rf = bench.roofline(prof, 1, peaks, "measured", timed_s=0.09, clk=full)
    assert rf["peak"] == 1636.3 and "burst" in rf["peak_source"]
    assert abs(rf["frac"] - rf["achieved"] / 1636.3) < 1e-3
    # a long region, or a clock held below its maximum, keeps the sustained figure
    assert bench.roofline(prof, 1, peaks, "measured", timed_s=4.0, clk=full)["peak"] == 1375.0
    low = {"sm_mhz": 1312.0, "sm_max_mhz": 1965}
    assert bench.roofline(prof, 1, peaks, "measured", timed_s=0.09, clk=low)["peak"] == 1375.0
    assert bench.roofline(prof, 1, peaks, "measured", timed_s=0.09, clk=None)["peak"] == 1375.0


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier()
        got = bench.max_over_ranks(10.0 + 5.0 * rank)
        q.put((rank, got, bench.dist_env()))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [15.0, 15.0]
    assert [r[2][0] for r in res] == [0, 1] and all(r[2][2] == 2 for r in res)


def test_single_process_reduction_is_identity():
    assert bench.max_over_ranks(3.25) == 3.25


def test_kernel_classes_of_ncu_names():
    kc = bench.kernel_class
    assert kc("void qnf4::nf4_linear_gemm_kernel<qnf4::NF4WCfg<false, 2>>(CUtensorMap_st, ...)")[0] == "fwd_gemm"
    assert kc("void qnf4::nf4_linear_gemm_kernel<qnf4::NF4WCfg<true, 2>>(CUtensorMap_st, ...)")[0] == "bwd_gemm"
    assert kc("void qnf4::nf4_linear_gemm_kernel<qnf4::NF4WCfg<1, 2>>(...)")[0] == "bwd_gemm"
    assert kc("void qnf4::nf4_expand_scales_kernel<true>(const unsigned char *, ...)")[0] == "fwd_gemm"
    assert kc("void qnf4::nf4_expand_scales_kernel<0>(const unsigned char *, ...)")[0] == "bwd_gemm"
    for k in ("nf4_quantize_pass1<float>(const T1 *)", "nf4_mean(const double *)", "nf4_dq_pass2(const float *)"):
        assert kc("void qnf4::" + k)[0] == "quantize"
    assert kc("void qnf4::nf4_dequantize_kernel<1, 0>(const unsigned char *)")[0] == "dequantize"
    cls, label = kc("void qnf4::gemm_sm100_kernel<qnf4::GemmCfg<64, false, false, 3>>(CUtensorMap_st)")
    assert cls is None and label == "gemm_sm100_kernel"


def test_ncu_summary_writes_per_call_traffic(tmp_path, capsys):
    """A hand-made launch list: two timed calls of each class, one extra kernel outside the classes."""
    rows = [["ID", "Kernel Name", "Metric Name", "Metric Unit", "Metric Value"]]
    names = ["void qnf4::nf4_expand_scales_kernel<1>(x)", "void qnf4::nf4_linear_gemm_kernel<qnf4::NF4WCfg<0, 2>>(x)",
             "void qnf4::split_reduce_kernel<0>(x)"] * 2
    for i, n in enumerate(names):
        rows += [[str(i), n, "gpu__time_duration.sum", "us", "10"],
                 [str(i), n, "dram__bytes_read.sum", "Mbyte", str(1 + i)],
                 [str(i), n, "dram__bytes_write.sum", "byte", "1000"]]
    csv_path = tmp_path / "launches.csv"
    csv_path.write_text("\n".join(",".join(f'"{c}"' for c in r) for r in rows) + "\n")
    out = tmp_path / "traffic.json"
    assert bench.ncu_summary(str(csv_path), 6, 2, "cmd", str(out)) == 0
    import json
    t = json.loads(out.read_text())
    # fwd_gemm launches are ids 0, 1, 3, 4: (1 + 2 + 4 + 5) MB read + 4 x 1000 B written, over 2 calls
    assert t["fwd_gemm"]["bytes_per_launch"] == round((12e6 + 4000) / 2)
    assert t["fwd_gemm"]["source_hash"] == bench.source_hash("fwd_gemm") and t["fwd_gemm"]["command"] == "cmd"
    assert set(t) == {"fwd_gemm"}
    assert "6 launches" in capsys.readouterr().out
