"""Host-side helpers of bench.py (CPU): the kernel-source key of the recorded ncu traffic
and the workload arithmetic the roofline divides by."""
import json
import os
import re
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _strip(src):
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def test_kernel_hash_ignores_comments_and_layout():
    h0 = bench.kernel_source_hash()
    assert re.fullmatch(r"[0-9a-f]{16}", h0)
    # the hash sees the same token stream whatever the comments and blank space say
    csrc = os.path.join(ROOT, "bit_recurrent_state_lores_b200", "csrc")
    a = open(os.path.join(csrc, "lores_step.cuh")).read()
    assert _strip(a) == _strip("/* note */\n" + a.replace("\n", "\n\n") + "\n// trailing\n")
    assert _strip(a) != _strip(a.replace("kFull", "kFull2", 1))


def test_traffic_record_names_the_current_kernel_or_is_ignored():
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for key, e in rec.items():
        assert {"kernel_hash", "dram_read", "dram_write"} <= set(e)
        assert e["dram_bytes_per_launch"] == e["dram_read"] + e["dram_write"]


def test_tile_and_launch_bytes_of_the_default_workload():
    from bit_recurrent_state_lores_b200 import synth
    wl = synth.workload("sweep", B=256, layers=1)
    # 128x128 int8 codes + one fp32 scale per row, read and written; q, k (d_k), v (d_v),
    # alpha, beta read; o (d_v) written
    codes, scales = 128 * 128, 128 * 4
    assert (wl.d_k, wl.d_v, wl.G) == (128, 128, 128)
    assert bench.tile_bytes(wl, 8) == 2 * (codes + scales) + (3 * 128 + 2) * 4 + 128 * 4 == 35848
    assert bench.tile_bytes(wl, 4) == 19464
    assert bench.tile_bytes(wl, 32) == 2 * 4 * codes + (3 * 128 + 2) * 4 + 128 * 4 == 133128
    assert bench.launch_bytes(wl, [8] * 32) == 256 * 32 * 35848 == 293666816


def test_reference_arm_runs_the_oracle_without_the_gpu_library():
    """The CPU arm times the oracle on all host cores and never loads liblores.so."""
    import subprocess
    code = (
        "import sys, json, runpy, io, contextlib\n"
        "sys.argv = ['bench.py', '--impl', 'reference', '--steps', '2', '--warmup', '1']\n"
        "buf = io.StringIO()\n"
        "with contextlib.redirect_stdout(buf):\n"
        "    runpy.run_path('bench.py', run_name='__main__')\n"
        "line = json.loads(buf.getvalue().strip().splitlines()[-1])\n"
        "print(json.dumps({'line': line, 'loaded': 'bit_recurrent_state_lores_b200.lores' in sys.modules}))\n")
    out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                         timeout=600, check=True).stdout
    res = json.loads(out.strip().splitlines()[-1])
    assert res["loaded"] is False
    line = res["line"]
    assert line["impl"] == "reference" and line["value"] > 0
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["affinity_cores"] >= 1
    assert cb["cpu_model"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0
