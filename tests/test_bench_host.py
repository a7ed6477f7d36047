"""Host-side pieces of bench.py that need no GPU: the reference arm's JSON line
(the oracle timed on the host cores) and the byte accounting both arms share."""
import json
import os
import subprocess
import sys

import bench
import qwm_synth as syn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_packed_bytes_per_token_head():
    # 2 x (d/4 codes + 4 d/G group parameters + index) + r coefficients + 2 scale bytes
    assert bench.packed_bytes_per_token_head(syn.get_config("480p")) == 108
    assert bench.packed_bytes_per_token_head(syn.get_config("720p")) == 110
    tiny = syn.get_config("tiny")
    assert bench.packed_bytes_per_token_head(tiny) == 2 * (16 + 16 + 1) + 4 + 2


def test_config_dict_names_workload_l2_and_parallelism():
    c = syn.get_config("480p")
    d = bench.config_dict(c, "w", 1, "replica", c.heads)
    assert set(d) == {"workload", "l2", "parallelism"}
    assert d["parallelism"] == "replicas x1"
    assert "162 MB" in d["l2"] and "larger" in d["l2"]
    d2 = bench.config_dict(c, "w", 4, "heads", 10)
    assert d2["parallelism"] == "heads split over 4 ranks (10 on rank 0)"


def test_reference_arm_line_on_the_host_cores():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "tiny",
                        "--steps", "1", "--warmup", "3"], cwd=ROOT, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["value"] > 0 and line["higher_is_better"]
    assert set(line["config"]) == {"workload", "l2", "parallelism"}
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert cb["host_cores"] == bench.host_cpu()[0] and cb["sample"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
