"""The reference arm of bench.py (`--impl reference`: the float64 oracle timed on
the host) prints one JSON line with the bench contract's keys; CPU only, a small
sample."""
import io
import json
from contextlib import redirect_stdout

import bench


def test_reference_arm_prints_one_contract_line():
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--workload", "tiny_f32", "--steps", "1",
                         "--warmup", "3", "--ref-seconds", "0.2"])
    assert rc == 0
    lines = [ln for ln in buf.getvalue().splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["value"] > 0 and d["unit"] == "channel-tokens/s" and d["higher_is_better"] is True
    assert d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    assert "tiny_f32" in d["config"]["workload"]
    # the same config dict as our arm, and on every host core
    assert d["config"] == bench.config_of(bench.WORKLOADS["tiny_f32"], 1, "auto")
    from oracle.timing import host_cores
    assert cb["cores"] == host_cores()


def test_reference_arm_loads_no_cuda_library():
    """The reference arm must not map the library it is compared with."""
    import subprocess
    import sys
    code = ("import bench, sys; bench.main(['--impl', 'reference', '--workload', 'tiny_f32', "
            "'--steps', '1', '--warmup', '3', '--ref-seconds', '0.1']); "
            "maps = open('/proc/self/maps').read(); "
            "sys.exit(3 if 'librglru_b200' in maps else 0)")
    r = subprocess.run([sys.executable, "-c", code], cwd=bench.ROOT, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]


def test_bench_refuses_fewer_than_three_warmups():
    import pytest
    with pytest.raises(SystemExit):
        bench.main(["--impl", "reference", "--warmup", "2"])
