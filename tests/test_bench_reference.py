"""bench.py's reference arm (the CPU oracle on bounded samples) runs without a GPU and
prints one JSON line with the fields the measurement contract names."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--config", "tiny", "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT, check=True)
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["unit"] == "tokens/s" and line["value"] > 0 and line["higher_is_better"] is True
    assert line["n_gpus"] == 1 and line["steps"] == 1 and line["warmup"] == 0
    assert line["config"]["workload"] == "tiny"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_kernel_records_are_keyed_to_code_not_comments():
    """bench.source_hash ignores comments and layout (a comment edit keeps a kernel's ncu
    record), but any change of code tokens changes it; and every committed traffic record
    names a kernel bench.py knows."""
    sys.path.insert(0, ROOT)
    import bench
    a = "int f(int x) {  // one\n  return x + 1; /* two\n lines */ }\n"
    b = "int f(int x)\n{\n    return x + 1;   // another comment\n}"
    c = "int f(int x) { return x + 2; }"
    assert bench.code_tokens(a) == bench.code_tokens(b) == "int f(int x) { return x + 1; }"
    assert bench.code_tokens(c) != bench.code_tokens(a)
    for name in os.listdir(os.path.join(ROOT, "profiles")):
        if name.endswith("_traffic.txt"):
            kernel = name[: -len("_traffic.txt")]
            assert kernel in bench.KERNEL_SOURCES, kernel
            kv = dict(l.split(":", 1) for l in open(os.path.join(ROOT, "profiles", name))
                      if ":" in l and not l.startswith("#"))
            assert len(kv["source_sha"].strip()) == 16 and int(kv["dram_bytes_per_launch_full"]) > 0
