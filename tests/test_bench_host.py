"""bench.py's host-side logic without a GPU: workload overrides, the
algorithmic bytes and flops per stage, and the traffic record keyed to the
GEMM source's hash."""
import hashlib
import os
import sys

import bench
from workloads import CONFIGS


def _args(**kw):
    old = sys.argv
    sys.argv = ["bench.py"] + [a for k, v in kw.items() for a in
                               ((f"--{k.replace('_', '-')}",) if v is True else (f"--{k.replace('_', '-')}", str(v)))]
    try:
        return bench.parse()
    finally:
        sys.argv = old


def test_shape_overrides():
    sh = bench.shape_of(_args(config="mixtral"))
    assert (sh.T, sh.d, sh.E, sh.k, sh.F) == (4096, 4096, 8, 2, 14336)
    sh1 = bench.shape_of(_args(config="mixtral", k=1, combine_in_gemm=True))
    assert sh1.k == 1 and sh1.name.endswith("_k1") and sh1.d == 4096
    shr = bench.shape_of(_args(config="mixtral", T=512, F=4096))
    assert (shr.T, shr.F) == (512, 4096) and shr.name != "mixtral"


def test_algorithmic_bytes_and_flops():
    sh = CONFIGS["mixtral"]
    kept = [1024] * 8                       # R = 8192 rows, all experts active
    a = bench.algorithmic(sh, kept)
    T, d, E, k, F, b = 4096, 4096, 8, 2, 14336, 2
    R = 8192
    assert a["route"]["bytes"] == T * d * b + d * E * b + T * k * 8
    assert a["gather"]["bytes"] == T * d * b + R * d * b
    assert a["ffn_up"]["flops"] == 2 * R * d * F * 2
    assert a["ffn_up"]["bytes"] == E * d * F * b * 2 + R * d * b + R * F * b
    assert a["ffn_down"]["flops"] == 2 * R * F * d
    assert a["combine"]["bytes"] == R * d * b + T * k * 8 + T * d * b
    # an expert with no rows reads no weights
    a7 = bench.algorithmic(sh, [0] + [1024] * 7)
    assert a7["ffn_down"]["bytes"] == 7 * F * d * b + 7168 * F * b + 7168 * d * b
    a6 = bench.algorithmic(sh, [0, 0] + [1365] * 6)
    assert a6["ffn_down"]["bytes"] == 6 * F * d * b + 8190 * F * b + 8190 * d * b


def test_algorithmic_combine_in_gemm_counts_zeroed_rows():
    sh = CONFIGS["mixtral"].with_(k=1, cf=1.0)
    kept = [500] * 8                        # 4000 of 4096 tokens kept, 96 dropped
    a = bench.algorithmic(sh, kept, combine_in_gemm=True)
    b = bench.algorithmic(sh, kept)
    assert a["gather"]["bytes"] - b["gather"]["bytes"] == 96 * 4096 * 2


def test_traffic_record_matches_source_hash():
    src = os.path.join(bench.ROOT, "mixture_experts_routing_route_b200", "csrc", "gemm_sm100.cu")
    with open(src, "rb") as f:
        h = hashlib.sha256(f.read()).hexdigest()[:16]
    rec = {}
    with open(bench.TRAFFIC_FILE) as f:
        for line in f:
            parts = line.split()
            if parts and not line.startswith("#"):
                rec[(parts[0], parts[1])] = (int(parts[2]), parts[3])
    t = bench.measured_traffic("grouped_gemm_up_swiglu", "mixtral")
    if rec[("grouped_gemm_up_swiglu", "mixtral")][1] == h:
        assert t == rec[("grouped_gemm_up_swiglu", "mixtral")][0]
    else:
        assert t is None                     # a changed kernel reports no stale traffic
    assert bench.measured_traffic("grouped_gemm_up_swiglu", "no_such_workload") is None


def test_reference_arm_never_loads_the_library_and_shares_the_config():
    """The reference arm (the CPU oracle) runs in a process that maps no
    library .so of this repository, and prints the config the GPU arm prints
    for the same flags."""
    import json
    import subprocess
    code = (
        "import sys, json, io, contextlib\n"
        "sys.argv = ['bench.py', '--impl', 'reference', '--config', 'tiny_fp32', '--steps', '1',"
        " '--warmup', '0']\n"
        "import bench\n"
        "buf = io.StringIO()\n"
        "with contextlib.redirect_stdout(buf):\n"
        "    bench.main()\n"
        "maps = open('/proc/self/maps').read()\n"
        "print(json.dumps({'line': json.loads(buf.getvalue().strip().splitlines()[-1]),"
        " 'pkg': 'mixture_experts_routing_route_b200' in sys.modules,"
        " 'so': 'libmoe_b200' in maps}))\n")
    res = subprocess.run([sys.executable, "-c", code], cwd=bench.ROOT, capture_output=True, text=True,
                         timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    got = json.loads(res.stdout.strip().splitlines()[-1])
    assert not got["pkg"] and not got["so"]
    line = got["line"]
    assert line["impl"] == "reference" and line["unit"] == "tokens/s"
    args = _args(config="tiny_fp32")
    assert line["config"] == json.loads(json.dumps(bench.arm_config(bench.shape_of(args), args, 1)))


def test_stage_roofline_and_dispatch_span():
    sh = CONFIGS["mixtral"]
    args = _args()
    alg = bench.algorithmic(sh, [1024] * 8)
    stage_ms = {"route": 0.0201, "permute": 0.0103, "gather": 0.0226, "ffn_up": 1.5, "ffn_down": 0.85,
                "combine": 0.019}
    peaks = {"hbm_gbs": 6546.9, "bf16_tflops": 1676.5}
    roof = bench.stage_roofline(sh, stage_ms, alg, peaks, 1676.5, args)
    assert abs(roof["route"]["GB_s"] - alg["route"]["bytes"] / 20.1e-6 / 1e9) < 1e-6
    assert abs(roof["ffn_up"]["tensor_frac"] - alg["ffn_up"]["flops"] / 1.5e-3 / 1e12 / 1676.5) < 1e-12
    span = bench.dispatch_span_of(stage_ms, alg, peaks)
    byts = alg["route"]["bytes"] + alg["permute"]["bytes"] + alg["gather"]["bytes"]
    assert abs(span["us"] - 53.0) < 1e-9
    assert abs(span["hbm_frac"] - byts / 53.0e-6 / 1e9 / 6546.9) < 1e-12
