"""Host-side checks of bench.py that need no GPU: the reference arm (the oracle on the host
cores) prints one JSON line with the measurement contract's keys, and under a multi-rank
launch only rank 0 runs it."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(args, extra_env=None, timeout=600):
    env = dict(os.environ)
    env.pop("RANK", None)
    env.pop("WORLD_SIZE", None)
    env.pop("LOCAL_RANK", None)
    env.update(extra_env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=timeout)


def test_reference_arm_json_line(orc):
    r = _bench(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0.0
    assert d["steps"] == 1 and d["warmup"] == 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] and d["data"] == "synthetic"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    assert d["sweep"]["unit"] == "blocks/s" and d["sweep"]["value"] > 0.0


def test_reference_arm_other_ranks_exit_without_work():
    r = _bench(["--impl", "reference", "--steps", "1", "--warmup", "0", "--gpus", "2"],
               {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}, timeout=120)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_record_traffic_reads_both_ncu_csv_forms(tmp_path, monkeypatch):
    """bench.py --record-traffic: DRAM bytes of a row's kernel from an ncu CSV log, in the
    one-row-per-metric form (ncu --csv --metrics) and the one-row-per-launch form
    (ncu -i REP --csv --page raw --metrics), averaged over the captured calls, with the
    case's units and the hash of the sources; the bench scales bytes per unit."""
    import json

    import bench

    per_metric = tmp_path / "a.csv"
    per_metric.write_text(
        '==PROF== Connected\n'
        '"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size","Grid Size",'
        '"Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"\n'
        '"0","1","p","h","void amax_kernel<0>(AmaxParams)","1","7","(512, 1, 1)","(592, 1, 1)","0","10.0",'
        '"Command line profiler metrics","dram__bytes_read.sum","Mbyte","939.68"\n'
        '"0","1","p","h","void amax_kernel<0>(AmaxParams)","1","7","(512, 1, 1)","(592, 1, 1)","0","10.0",'
        '"Command line profiler metrics","dram__bytes_write.sum","byte","2000"\n')
    per_launch = tmp_path / "b.csv"
    per_launch.write_text(
        '"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size","Grid Size",'
        '"Device","CC","dram__bytes_read.sum","dram__bytes_write.sum"\n'
        '"","","","","","","","","","","","Mbyte","Mbyte"\n'
        '"0","1","p","h","cast_kmax_kernel(CastParams)","1","7","(512, 1, 1)","(256, 1, 1)","0","10.0","8.0","0"\n'
        '"1","1","p","h","cast_rewrite_kernel(CastParams)","1","7","(256, 1, 1)","(296, 1, 1)","0","10.0","140.0","100.0"\n')
    out = tmp_path / "profiles"
    out.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    csrc = tmp_path / "nvfp4_block_numerics_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in ("quant.cu", "nv4_common.cuh", "cast.cu"):
        (csrc / f).write_text(f"// {f}\n")
    bench.record_traffic([f"tensor_amax={per_metric}", f"mxfp4_to_nvfp4={per_launch}"])
    doc = json.loads((out / "dram_traffic.json").read_text())["kernels"]
    assert doc["tensor_amax"]["dram_read_bytes"] == 939680000 and doc["tensor_amax"]["dram_write_bytes"] == 2000
    assert doc["mxfp4_to_nvfp4"]["dram_read_bytes"] == 148000000      # both kernels of one call
    assert doc["mxfp4_to_nvfp4"]["dram_write_bytes"] == 100000000
    t = bench.traffic_table()
    assert abs(t["tensor_amax"] - 939682000 / (65536 * 7168)) < 1e-9
    (csrc / "quant.cu").write_text("// changed\n")                  # a changed kernel drops its entry
    assert "tensor_amax" not in bench.traffic_table() and "mxfp4_to_nvfp4" in bench.traffic_table()
