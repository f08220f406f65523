"""Host-side checks of bench.py: metric accounting, the reference (CPU
oracle) arm, and the multi-rank plumbing on world_size-2 gloo process groups
(no GPU needed)."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
import workloads as W  # noqa: E402


def test_metric_value_units_and_world_scaling():
    prob = W.Problem("dense", 64, 2112, 7168, 1, None, None, 0, None, None)
    gbps = bench.metric_value(prob, "GB/s", 0.01, 1)
    assert abs(gbps - prob.bytes() / 1e-5 / 1e9) < 1e-6
    assert abs(bench.metric_value(prob, "GB/s", 0.01, 4) - 4 * gbps) < 1e-6
    tf = bench.metric_value(prob, "TFLOP/s", 0.01, 2)
    assert abs(tf - 2 * prob.flops() / 1e-5 / 1e12) < 1e-6


def test_rank_problems_share_shapes_not_values():
    p0, p1 = bench.rank_problem("dense_tiny", 0), bench.rank_problem("dense_tiny", 1)
    assert p0.a.shape == p1.a.shape and p0.b.shape == p1.b.shape
    assert not np.array_equal(p0.a, p1.a)


def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "dense_tiny", "--steps", "1", "--warmup", "3"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["cpu_baseline"]["kind"] == "oracle"
    assert d["cpu_baseline"]["cores"] >= 1 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["unit"] == d["unit"]
    assert d["config"]["workload"] == "dense_tiny"


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "dense_tiny", "--steps", "1", "--warmup", "3"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks([1.0 + rank, 5.0 - rank], "cpu", world)
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world_2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res[0] == res[1] == [2.0, 5.0]


def test_every_workload_has_a_unit_a_kernel_and_a_config():
    """Every bench workload resolves to a unit, a profiled kernel name with
    hashed sources, and a JSON-serialisable shape config; other ranks draw
    other values of the same shapes."""
    names = (list(W.WORKLOADS) + list(W.QUANT_WORKLOADS) + list(W.BF16_WORKLOADS) + list(W.FFN_WORKLOADS))
    small = {"quant_tiny", "bf16_dense_decode_m64", "dense_tiny", "dense_decode_m64"}
    for w in names:
        assert w in bench.UNIT, w
        k = bench.kernel_name(w)
        assert k in bench.KERNEL_SOURCES and len(bench.kernel_source_hash(k)) == 16
        if w not in small:
            continue
        p0, p1 = bench.rank_problem(w, 0), bench.rank_problem(w, 1)
        cfg = bench.shape_config(p0)
        json.dumps(cfg)
        assert cfg == bench.shape_config(p1)
        assert p0.bytes() > 0
        a0 = p0.x if hasattr(p0, "x") else p0.a
        a1 = p1.x if hasattr(p1, "x") else p1.a
        assert not np.array_equal(a0, a1)


@pytest.mark.parametrize("workload", ["quant_tiny", "bf16_dense_decode_m64"])
def test_reference_arm_for_the_next_rows(workload):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", workload, "--steps", "1", "--warmup", "3"],
                       cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["config"]["workload"] == workload
    assert d["value"] > 0 and d["unit"] == bench.UNIT[workload]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


@pytest.mark.parametrize("workload,launches,graph", [("dense_decode_m64", 1, False), ("masked_g16", 1, True),
                                                     ("ffn_g4", 2, False), ("quant_tokens_32768", 1, False)])
def test_our_json_line_carries_every_contract_key(monkeypatch, capsys, workload, launches, graph):
    """The line of our arm, assembled from a stubbed device run: every key the
    bench contract names is present, with the roofline fraction, the launch
    count and (masked GEMMs only) the CUDA-graph figure consistent; the
    workload config holds no measurement."""
    prob = bench.rank_problem(workload, 0)
    clocks = {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": [], "samples": 40}
    head = bench.Timing(workload, prob, 0.5, 0.49, launches)
    monkeypatch.setattr(bench, "run_ours",
                        lambda args, rank, world, lr: (head, 0.8, 100, 20, 0.51 if graph else 0.0, [],
                                                       clocks, 0.0))
    monkeypatch.setattr(sys, "argv", ["bench.py", "--workload", workload, "--steps", "7", "--warmup", "3",
                                      "--no-cpu-baseline"])
    assert bench.main() == 0
    out = [l for l in capsys.readouterr().out.splitlines() if l.strip()]
    assert len(out) == 1
    line = json.loads(out[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches",
                "clocks", "measurement"):
        assert key in line, key
    assert line["config"] == {"workload": workload, **bench.shape_config(prob)}
    assert not set(line["config"]) & {"l2", "tflops", "gbps", "ms_median_step"}
    assert line["scaling"] == "weak"
    roof = line["roofline"]
    for key in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert key in roof, key
    assert abs(roof["frac"] - roof["achieved"] / roof["peak"]) < 1e-12
    assert set(line["e2e"]) >= {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"}
    assert line["e2e"]["value"] < line["value"]          # the e2e step (0.8 ms) is slower than 0.5 ms
    assert line["gpu_launches"] == 7 * launches
    assert ("graph" in line) == graph
    assert line["clocks"] == clocks
    assert "shapes" not in line


def test_default_run_is_the_contiguous_prefill_with_every_shape(monkeypatch, capsys):
    """With no flags the headline is the largest configuration (the contiguous
    MoE prefill) and ``shapes`` carries every configuration of the benchmark set,
    each with its own roofline entry; the reference arm names the same config."""
    assert bench.DEFAULT_WORKLOAD == "contiguous_g4"
    assert set(bench.SHAPES) == {"dense_tiny", "dense_decode_m64", "dense_decode_m128", "dense_large",
                                 "contiguous_g4", "masked_g16"}
    tiny = bench.rank_problem("dense_tiny", 0)
    probs = {w: tiny for w in bench.SHAPES}     # stand-in problems: the accounting is per workload

    def fake(args, rank, world, lr):
        assert args.shape_list == list(bench.SHAPES)
        shapes = [bench.Timing(w, probs[w], 0.01 * (i + 1), 0.01, 1) for i, w in enumerate(args.shape_list)]
        head = shapes[args.shape_list.index("contiguous_g4")]
        return head, 0.9, 10, 10, 0.0, shapes, {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}, 0.006
    monkeypatch.setattr(bench, "run_ours", fake)
    monkeypatch.setattr(sys, "argv", ["bench.py", "--steps", "5", "--warmup", "3", "--no-cpu-baseline"])
    assert bench.main() == 0
    line = json.loads(capsys.readouterr().out.strip())
    assert line["config"]["workload"] == "contiguous_g4"
    assert set(line["shapes"]) == set(bench.SHAPES)
    for w, e in line["shapes"].items():
        assert e["unit"] == bench.UNIT[w]
        assert set(e["roofline"]) >= {"achieved", "peak", "frac", "traffic"}
        assert abs(e["roofline"]["frac"] - e["roofline"]["achieved"] / e["roofline"]["peak"]) < 1e-12
    assert line["shapes"]["contiguous_g4"]["ms_per_step"] == line["ms_per_step"]
    assert "vs_pages" in line["shapes"]["dense_decode_m64"]
    assert line["vs_baseline"] is None            # no page row states all of M, N and K of this workload
    assert line["measurement"]["launch_floor_ms"] == 0.006


def test_rotating_graph_copies_exceed_twice_the_l2():
    """Decode-sized inputs get enough copies that together they exceed twice the
    L2, so every call of the rotating-graph timing reads from HBM; small and
    large inputs are not timed that way."""
    for w in ("dense_decode_m64", "dense_decode_m128"):
        prob = bench.rank_problem(w, 0)
        nbytes = sum(x.nbytes for x in (prob.a, prob.sfa, prob.b, prob.sfb))   # the call's host inputs
        sets = bench.rotation_sets(nbytes)
        assert sets >= 2 and (sets - 1) * nbytes > 2 * bench.L2_BYTES
    assert bench.rotation_sets(264224) == 0
    assert bench.rotation_sets(500 << 20) == 0
    t = bench.Timing("dense_decode_m64", bench.rank_problem("dense_decode_m64", 0), 0.015, 0.015, 1,
                     graph_ms=0.0105, graph_sets=18, graph_calls=50)
    e = bench.shape_entry(t, 1)["graph_rotating"]
    assert e["unit"] == "GB/s" and e["input_copies"] == 18 and e["ms_per_call"] == 0.0105
    assert abs(e["value"] - t.prob.bytes() / 0.0105e-3 / 1e9) < 1e-6 * e["value"]
    assert "vs_pages" in e


def test_headline_carries_its_rotating_graph_figure(monkeypatch, capsys):
    """A decode-sized headline (``--workload dense_decode_m64 --shapes none``)
    prints its rotating-graph figure at the top level."""
    prob = bench.rank_problem("dense_decode_m64", 0)
    head = bench.Timing("dense_decode_m64", prob, 0.015, 0.015, 1, graph_ms=0.0104, graph_sets=18, graph_calls=50)
    monkeypatch.setattr(bench, "run_ours", lambda a, r, w, lr: (head, 0.05, 10, 10, 0.0, [],
                                                                 {"sm_mhz": 1965, "sm_max_mhz": 1965,
                                                                  "reasons": []}, 0.0))
    monkeypatch.setattr(sys, "argv", ["bench.py", "--workload", "dense_decode_m64", "--shapes", "none",
                                      "--steps", "5", "--warmup", "3", "--no-cpu-baseline"])
    assert bench.main() == 0
    line = json.loads(capsys.readouterr().out.strip())
    assert line["graph_rotating"]["ms_per_call"] == 0.0104
    assert line["graph_rotating"]["value"] > line["value"]


def test_shape_selection():
    assert bench.parse_shapes("auto", "contiguous_g4") == list(bench.SHAPES)
    assert bench.parse_shapes("auto", "dense_large") == []
    assert bench.parse_shapes("none", "contiguous_g4") == []
    assert bench.parse_shapes("dense_tiny,masked_g16", "dense_large") == ["dense_tiny", "masked_g16"]
    with pytest.raises(SystemExit):
        bench.parse_shapes("dense_tiny,nope", "dense_large")


def test_traffic_comes_from_the_capture_file_only_while_the_sources_match(monkeypatch, tmp_path):
    """roofline.traffic is read from a machine-readable capture file keyed by
    kernel and workload, and only while the kernel sources hash to the value
    recorded with the capture."""
    f = tmp_path / "traffic.json"
    h = bench.kernel_source_hash("fp8_gemm_kernel")
    f.write_text(json.dumps({"captures": {
        "fp8_gemm_kernel/dense_large": {"kernel_source_hash": h, "dram_bytes_per_launch": 123.0},
        "fp8_gemm_kernel/masked_g16": {"kernel_source_hash": "0" * 16, "dram_bytes_per_launch": 5.0}}}))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.profiled_traffic("dense_large") == 123.0
    assert bench.profiled_traffic("masked_g16") is None           # stale capture
    assert bench.profiled_traffic("contiguous_g4") is None        # no capture
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.json"))
    assert bench.profiled_traffic("dense_large") is None
