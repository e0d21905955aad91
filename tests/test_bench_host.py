"""Host-side logic of bench.py on the CPU: the reference arm's JSON line, the
max-over-ranks timing and barrier over a two-rank gloo group, the launch
count and the committed-profile traffic lookup."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _json_lines(text):
    return [json.loads(l) for l in text.splitlines() if l.startswith("{")]


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    d = lines[0]
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"):
        assert k in d, k
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["value"] > 0
    assert d["config"]["workload"] == "480p_bidir"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_under_two_ranks_prints_once():
    port = _free_port()
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                        "--nproc-per-node", "2", "--master-addr", "127.0.0.1", "--master-port",
                        str(port), "bench.py", "--impl", "reference", "--gpus", "2", "--steps",
                        "1", "--warmup", "0"], cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1 and lines[0]["n_gpus"] == 2


def _rank_main(rank, port, values, out):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank,
                            world_size=2)
    bench.barrier(dist)
    out[rank] = bench.reduce_max(values[rank], dist)
    bench.barrier(dist)
    dist.destroy_process_group()


def test_reduce_max_and_barrier_over_gloo():
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(port, [1.5, 4.25], out), nprocs=2, join=True)
        assert dict(out) == {0: 4.25, 1: 4.25}


def test_reduce_max_without_group_is_identity():
    assert bench.reduce_max(3.0, None) == 3.0


def test_launches_per_forward():
    W = workloads.WORKLOADS
    assert bench.launches_per_forward(W["480p_bidir"], "bidirectional") == 2
    assert bench.launches_per_forward(W["480p_block_causal"], "block_causal") == 3
    assert bench.launches_per_forward(W["720p_long"], "block_causal") == 3
    # token-causal: two kernels on the tensor cores (bf16, D = 64), three on CUDA cores
    assert bench.launches_per_forward(W["480p_bidir"], "token_causal") == 2
    assert bench.launches_per_forward(W["tiny_f32"], "token_causal") == 3


def test_profile_traffic_lookup_is_tied_to_the_sources(tmp_path, monkeypatch):
    # a committed line counts only while its source hash matches the kernels
    h = bench.kernel_source_hash()
    assert len(h) == 12
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    csrc = tmp_path / "linear_attention_video_relu_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("// kernel\n")
    h2 = bench.kernel_source_hash()
    (tmp_path / "profiles" / "x.txt").write_text(
        "# bench-traffic apply 480p_bidir 123 %s\n# bench-traffic apply 720p_long 9 %s\n"
        "# bench-traffic state_build 480p_bidir 77 000000000000\n" % (h2, h2))
    assert bench.ncu_traffic("apply", "480p_bidir") == 123
    assert bench.ncu_traffic("apply", "720p_long") == 9
    assert bench.ncu_traffic("state_build", "480p_bidir") is None
    # comments do not count; code does
    (csrc / "k.cu").write_text("/* a\n note */ // kernel, reworded\n")
    assert bench.kernel_source_hash() == h2
    (csrc / "k.cu").write_text("// kernel\nint x;\n")
    assert bench.kernel_source_hash() != h2
    assert bench.ncu_traffic("apply", "480p_bidir") is None


def test_committed_profiles_name_their_command():
    pdir = os.path.join(ROOT, "profiles")
    names = [n for n in os.listdir(pdir) if n.endswith((".txt", ".md"))]
    assert names
    for n in names:
        text = open(os.path.join(pdir, n)).read()
        assert "ncu " in text and "bench.py" in text, n
        assert len(text) < 8192, n


def test_secondary_lines_record_errors(monkeypatch):
    # a failing secondary line is reported with its error; the others still run
    calls = []

    def ok(*a, **k):
        calls.append(a[0] if a else None)
        return {"workload": "ok"}

    def boom(*a, **k):
        raise RuntimeError("device status after timing: bounded wait gave up")

    monkeypatch.setattr(bench, "measure_workload", ok)
    monkeypatch.setattr(bench, "measure_cross", boom)
    monkeypatch.setattr(bench, "measure_tconv", ok)
    monkeypatch.setattr(bench, "measure_block_steps", ok)
    lines = bench.secondary_lines(20, None, 6535.7, "measured")
    errs = [l for l in lines if "error" in l]
    assert len(errs) == 1 and errs[0]["w"] == "480p_bidir_x_text300/cross"
    assert "bounded wait" in errs[0]["error"]
    assert len(lines) == 9 and sum(1 for l in lines if l.get("w") == "ok") == 8


def test_secondary_lines_are_short():
    # every secondary result is reduced to a few short keys, so that ten of
    # them fit in the last ~3 KB of the bench output
    kern = lambda us, f, t=None: {"avg_us": us, "frac": f, "kernel": "x", "bound": "hbm",
                          "achieved": 1.0, "peak": 6535.7, "unit": "GB/s", "traffic": t,
                          "algorithmic_bytes": 1, "peak_source": "measured"}
    full = {"workload": "720p_long", "mode": "block_causal", "ms_per_step": 0.69123456,
            "tokens_per_s": 319876543.21, "hbm_gbs": 5234.5678, "hbm_frac": 0.80098765,
            "kernels": {"state_build": kern(350.123, 0.7712), "reduce_us": 14.2,
                        "apply": kern(320.5, 0.8123)}}
    c = bench.compact(full)
    assert c["w"] == "720p_long" and c["mode"] == "block_causal"
    assert c["ms"] == 0.6912 and c["frac"] == 0.801 and c["sb"] == [350.123, 0.7712, None]
    assert c["ap"] == [320.5, 0.8123, None] and c["red_us"] == 14.2
    cross = {"workload": "480p_bidir_x_text300", "mode": "cross", "n_kv": 300,
             "us_per_forward": 61.66, "tokens_per_s": 5.3e8, "algorithmic_bytes": 1,
             "hbm_gbs": 4392.1, "hbm_frac": 0.672}
    blk = {"workload": "720p_long_block_step", "block_tokens": 3680, "us_per_block": 30.9,
           "issue_us": 18.234, "tokens_per_s": 1.19e8, "hbm_frac": 0.2986}
    lines = [bench.compact(r) for r in (full, cross, blk)]
    assert lines[1]["us"] == 61.66 and lines[2]["us_blk"] == 30.9
    assert lines[2]["issue_us"] == 18.23
    full["kernels"]["apply"] = kern(320.5, 0.8123, 272841984)
    assert bench.compact(full)["ap"] == [320.5, 0.8123, 272.8]
    assert bench.compact(dict(cross, traffic=270900000))["traffic_MB"] == 270.9
    assert all(len(json.dumps(l)) < 200 for l in lines)


def test_only_selects_one_secondary_job():
    names = [n for n, _ in bench.secondary_jobs(5, None, 6535.7, "measured")]
    assert len(names) == len(set(names)) == 9
    for n in ("480p_bidir_x_text300/cross", "480p_hidden_tconv", "480p_2b_d112/bidirectional",
              "480p_bidir/token_causal"):
        assert n in names


def test_traffic_of_the_temporal_conv_follows_its_own_source(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    csrc = tmp_path / "linear_attention_video_relu_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "tc.cuh").write_text("int a;\n")
    (csrc / "tconv.cu").write_text("int b;\n")
    ht, hc = bench.kernel_source_hash("tconv"), bench.kernel_source_hash()
    assert ht != hc
    (tmp_path / "profiles" / "t.txt").write_text(
        "# bench-traffic temporal_conv 480p_hidden_tconv 300 %s\n" % ht)
    assert bench.ncu_traffic("temporal_conv", "480p_hidden_tconv") == 300
    (csrc / "tc.cuh").write_text("int a; int c;\n")      # other kernels change: still valid
    assert bench.ncu_traffic("temporal_conv", "480p_hidden_tconv") == 300
    (csrc / "tconv.cu").write_text("int b; int d;\n")    # its own source changes: stale
    assert bench.ncu_traffic("temporal_conv", "480p_hidden_tconv") is None


def test_every_committed_traffic_line_names_a_workload_the_bench_reads():
    # a '# bench-traffic <kernel> <workload> ...' line is only read back if its
    # workload key is one the bench looks up: the bare name for bidirectional
    # forwards, name/mode for the other modes, the cross and conv names
    import glob
    import os
    import bench
    keys = {"480p_bidir"}
    for name, _ in bench.secondary_jobs(1, None, 1.0, "measured"):
        if "/" in name:
            w, mode = name.split("/")
            keys.add(w if mode in ("bidirectional", "cross") else name)
        else:
            keys.add(name)
    seen = 0
    for path in glob.glob(os.path.join(bench.ROOT, "profiles", "*.txt")):
        for line in open(path):
            parts = line.split()
            if len(parts) == 6 and parts[:2] == ["#", "bench-traffic"]:
                seen += 1
                assert parts[2] in ("state_build", "apply", "temporal_conv"), (path, line)
                assert parts[3] in keys, (path, parts[3], sorted(keys))
    assert seen >= 10


def test_null_roofline_traffic_is_explained_once(monkeypatch):
    monkeypatch.setattr(bench, "ncu_traffic", lambda k, w: None)
    e = bench.roofline_entry("state_build", 268369920, [0.065, 0.066], 6535.7, "measured",
                             "480p_bidir")
    assert e["traffic"] is None
    assert abs(e["frac"] - 268369920 / 0.0655e-3 / 1e9 / 6535.7) < 1e-4
    note = bench.traffic_note({"roofline": e})
    assert bench.kernel_source_hash("tc") in note and len(note) < 60
    monkeypatch.setattr(bench, "ncu_traffic", lambda k, w: 273690112)
    e = bench.roofline_entry("state_build", 268369920, [0.065], 6535.7, "measured", "480p_bidir")
    assert e["traffic"] == 273690112 and bench.traffic_note({"roofline": e}) is None
