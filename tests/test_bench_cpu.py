"""The benchmark's output contract, checked on the CPU through its reference
arm (the oracle timed on host cores, no GPU needed): exactly one JSON line,
from rank 0 only, with the keys and types a benchmark driver reads."""
import json
import os
import socket
import subprocess
import sys

import pdssm_inputs as gen

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _lines(cmd, timeout=300):
    p = subprocess.run(cmd, capture_output=True, text=True, timeout=timeout, cwd=ROOT,
                       env=dict(os.environ, MASTER_ADDR="127.0.0.1"))
    assert p.returncode == 0, p.stderr[-3000:]
    return [ln for ln in p.stdout.splitlines() if ln.strip()]


def _check_line(d, n_gpus, steps, warmup):
    types = {"metric": str, "value": float, "unit": str, "n_gpus": int, "steps": int,
             "warmup": int, "ms_per_step": float, "higher_is_better": bool, "scaling": str,
             "dtype": str, "data": str, "config": dict, "cpu_baseline": dict, "e2e": dict}
    for key, typ in types.items():
        assert isinstance(d[key], typ), key
    assert d["impl"] == "reference"
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert (d["n_gpus"], d["steps"], d["warmup"]) == (n_gpus, steps, warmup)
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["config"]["workload"] == "tiny_fp32_select_fwd"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert cb["sample"]
    e = d["e2e"]
    assert (e["value"], e["unit"]) == (d["value"], d["unit"])
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_prints_one_contract_line():
    lines = _lines([sys.executable, "bench.py", "--impl", "reference", "--workload", "0",
                    "--steps", "2", "--warmup", "1"])
    assert len(lines) == 1
    _check_line(json.loads(lines[0]), 1, 2, 1)


def test_reference_arm_under_two_ranks_prints_once():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    lines = _lines([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                    "--nproc-per-node", "2", "--master-addr", "127.0.0.1", "--master-port",
                    str(port), "bench.py", "--impl", "reference", "--gpus", "2", "--workload",
                    "0", "--steps", "1", "--warmup", "1"])
    assert len(lines) == 1
    _check_line(json.loads(lines[0]), 2, 1, 1)


def test_l2_note_tells_resident_from_streamed_inputs():
    sys.path.insert(0, ROOT)
    import bench
    assert "larger than L2" in bench.l2_note(gen.workload(2))
    assert "larger than L2" in bench.l2_note(gen.workload(3))
    assert "fit in L2" in bench.l2_note(gen.workload(0))


def test_oracle_timing_on_one_and_several_threads():
    """The cpu_baseline leg: the oracle on one thread and on a thread pool
    over (batch, head) sequences; both count the same pieces of work."""
    sys.path.insert(0, ROOT)
    import bench
    cfg = gen.workload(4, B=1, H=4, L=600)
    inp = gen.generate(cfg)
    v1, s1, c1 = bench.time_oracle(cfg, inp, 30.0)
    v2, s2, c2 = bench.time_oracle(cfg, inp, 30.0, threads=3)
    assert v1 > 0 and v2 > 0 and (c1, c2) == (1, 3)
    # the whole small workload fits the budget: every sequence is timed once
    updates = cfg["B"] * cfg["H"] * cfg["L"] * cfg["N"]
    assert f"({updates} state updates" in s1 and f"({updates} state updates" in s2
    assert "single thread" in s1 and "3 threads" in s2
