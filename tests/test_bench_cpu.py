"""Host-side logic of bench.py without a GPU: the rank helpers over a
world_size-2 gloo group (barrier, max over ranks -- the only collectives the
replicas use), and the reference arm (the CPU oracle), including its
behaviour under torchrun where only rank 0 works and prints."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    r = bench.Ranks(backend="gloo")
    r.barrier()
    m = r.max(10.0 + 5.0 * rank)          # the slowest rank's time wins
    r.barrier()
    r.close()
    q.put((rank, m))


def test_ranks_barrier_and_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert got == [(0, 15.0), (1, 15.0)]


def _bench(args, env):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, cwd=ROOT,
                          env=dict(os.environ, **env), capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_one_json_line():
    r = _bench(["--impl", "reference", "--workload", "c0_small", "--steps", "2", "--warmup", "1",
                "--reference-seconds", "3"], {})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["config"]["workload"] == "c0_small"


def test_reference_arm_nonzero_rank_exits_without_work():
    r = _bench(["--impl", "reference", "--workload", "c0_small", "--steps", "2", "--warmup", "1",
                "--reference-seconds", "3"], {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_workload_accounting():
    sys.path.insert(0, ROOT)
    import bench
    c1 = bench.make_workload("c1_q_proj_480p")
    assert c1.flops() == 2.0 * 32760 * 5120 * 5120
    blk = bench.make_workload("c3_block_832x1104")
    step = bench.make_workload("c4_step_832x1104")
    # 8 hidden x hidden linears (two on 512 text tokens) + the FFN pair
    expect = 2.0 * (6 * 75348 * 5120 * 5120 + 2 * 512 * 5120 * 5120 + 2 * 75348 * 5120 * 13824)
    assert blk.flops() == pytest.approx(expect)
    assert step.flops() == pytest.approx(40 * expect)


def test_fused_accounting():
    """The fused FFN epilogue removes one quantization per block and writes
    E4M3 codes + scales instead of BF16 for ffn.net.0.proj."""
    sys.path.insert(0, ROOT)
    import bench
    M, H, F = 75348, 5120, 13824
    fused = bench.make_workload("c2_ffn_pair_832x1104")
    plain = bench.make_workload("c2_ffn_pair_832x1104", fused=False)
    assert fused.flops() == plain.flops()
    assert plain.quant_bytes() - fused.quant_bytes() == M * F * 3 + M * F // 32
    assert plain.gemm_bytes() - fused.gemm_bytes() == pytest.approx(M * F * (2 - (1 + 1 / 32)))
    bf = bench.make_workload("c3_block_832x1104")
    bp = bench.make_workload("c3_block_832x1104", fused=False)
    assert bp.quant_bytes() - bf.quant_bytes() == M * F * 3 + M * F // 32
    assert bf.flops() == bp.flops()


def test_per_linear_accounting_covers_the_step():
    """Every GEMM of a block is one named linear; their FLOPs add up to the
    workload's (so the per-linear rooflines cover the whole step), and the
    default workload is the 40-block step."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.parse([]).workload == "c4_step_832x1104"
    for fused in (True, False):
        for name in ("c3_block_832x1104", "c4_step_832x1104", "c2_ffn_pair_832x1104"):
            wl = bench.make_workload(name, fused=fused)
            per_block = sum(wl.linear_flops().values())
            blocks = getattr(wl, "nblocks", 1)
            assert blocks * per_block == pytest.approx(wl.flops()), (name, fused)
    assert bench.make_workload("c1_q_proj_480p").linear_flops() == {}


def test_both_arms_print_the_same_config():
    sys.path.insert(0, ROOT)
    import bench
    r = _bench(["--impl", "reference", "--workload", "c0_small", "--steps", "1", "--warmup", "1",
                "--reference-seconds", "2"], {})
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["config"] == bench.run_config(bench.make_workload("c0_small"), 1)


@pytest.mark.parametrize("scheme", ["fp8rowwise", "nvfp4"])
def test_reference_arm_other_schemes(scheme):
    r = _bench(["--impl", "reference", "--workload", "c0_small", "--scheme", scheme, "--steps", "2",
                "--warmup", "1", "--reference-seconds", "3"], {})
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads(r.stdout.strip().splitlines()[-1])
    assert d["impl"] == "reference" and d["value"] > 0 and d["config"]["scheme"]


def test_nvfp4_accounting():
    """NVFP4 moves 4-bit codes plus one scale byte per 16 elements."""
    sys.path.insert(0, ROOT)
    import bench
    wl = bench.make_workload("c1_q_proj_480p", scheme="nvfp4")
    M, K, N = 32760, 5120, 5120
    assert wl.flops() == 2.0 * M * N * K
    assert wl.quant_bytes() == M * K * 2 + M * K // 2 + M * K // 16
    assert wl.gemm_bytes() == pytest.approx((M + N) * K * 9 / 16 + 2 * M * N + 2 * N)
    # the 4-bit block-scaled kind: the FP4 peak is the BF16 figure x 4
    assert wl.tc_over_bf16 == bench.FP4_OVER_BF16 == 4.0 and wl.profile_kernel == "mxfp8_gemm"
    with pytest.raises(ValueError):
        bench.make_workload("c2_ffn_pair_832x1104", scheme="nvfp4")


def test_traffic_is_reported_only_for_the_profiled_kernel_files(tmp_path, monkeypatch):
    """roofline.traffic comes from profiles/<kernel>_<key>.json only while its
    hash equals the hash of that kernel's current source files."""
    sys.path.insert(0, ROOT)
    import bench
    from mxfp8_w8a8_quantized_b200 import build
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    kernel = "mxfp8_gemm"
    (prof / f"{kernel}_k.json").write_text(json.dumps(
        {"kernel_source_sha": build.source_sha(kernel), "dram_bytes_per_launch": 123}))
    assert bench.load_traffic("k", kernel) == 123
    (prof / f"{kernel}_k.json").write_text(json.dumps(
        {"kernel_source_sha": "0" * 16, "dram_bytes_per_launch": 123}))
    assert bench.load_traffic("k", kernel) is None
    assert bench.load_traffic("missing", "mxfp8_gemm") is None
    # the GEMM's hash covers its own files only; the library hash covers all
    assert build.source_sha("mxfp8_gemm") != build.source_sha()


def test_reference_arm_times_the_whole_chain():
    """For a chained workload the reference arm runs the oracle's chain
    (both FFN linears and the GELU), the workload the GPU arm times."""
    r = _bench(["--impl", "reference", "--workload", "c2_ffn_pair_832x1104", "--steps", "1", "--warmup", "1",
                "--reference-seconds", "4"], {})
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads(r.stdout.strip().splitlines()[-1])
    assert d["config"]["workload"] == "c2_ffn_pair_832x1104" and d["value"] > 0
    assert "FFN pair" in d["cpu_baseline"]["sample"]
