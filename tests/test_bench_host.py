"""Host-side pieces of the benchmark, checked without a GPU.

* the algorithmic work model that the roofline fields divide by (the scan's
  flops follow the causal prefix of every group; refine's bytes are its output
  rows, candidate rows and one read of q and k);
* DRAM traffic is taken from the committed one-head capture only while the
  refine source is the one that was captured, and scaled by the heads;
* the job throughput of a head-split layer and the clock-sample summary.
"""
import hashlib
import os
import shutil

import numpy as np

import bench
import synthetic


def test_algorithmic_work_at_l131072():
    c = synthetic.CONFIGS["C3"]
    alg = bench.algorithmic(c)
    L, H, d, g, k, Kc = c["L"], c["H"], c["d"], c["g"], c["top_k"], c["Kc"]
    # groups i = 0..L/g-1 scan the keys j < i*g + g - 1
    last = np.arange(0, L, g) + g - 1
    assert alg["scan_filter"] == ("tensor", 2.0 * d * H * float(last.sum()))
    assert abs(alg["scan_filter"][1] - 2.20e12) < 0.01e12
    n_cand = np.minimum(Kc, last)
    want = L * H * k * 4 + H * n_cand.sum() * 4 + 2 * L * H * d * 2
    assert alg["refine"] == ("hbm", float(want))
    assert abs(alg["refine"][1] - 20.4e9) < 0.1e9
    assert alg["proxy"][0] == "hbm" and alg["fallback"] == ("hbm", 0.0)


def test_traffic_follows_the_captured_source(tmp_path, monkeypatch):
    got = bench.measured_traffic("refine", 16)
    prof = os.path.join(bench.ROOT, "profiles", "refine_c3_one_head.md")
    fields = dict(line.split(": ", 1) for line in open(prof).read().splitlines() if ": " in line)
    per_head = float(fields["traffic_bytes_per_head_launch"])
    src = os.path.join(bench.ROOT, "query_group_top_b200", "csrc", "refine.cuh")
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if fields["source_sha256_16"].strip() == digest:
        assert got == per_head * 16
    else:
        assert got is None
    assert bench.measured_traffic("scan_filter", 16) is None
    # a changed kernel source voids the capture
    root = tmp_path / "repo"
    (root / "profiles").mkdir(parents=True)
    (root / "query_group_top_b200" / "csrc").mkdir(parents=True)
    shutil.copy(prof, root / "profiles" / "refine_c3_one_head.md")
    (root / "query_group_top_b200" / "csrc" / "refine.cuh").write_text("// another kernel\n")
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.measured_traffic("refine", 16) is None


def test_job_value_of_a_head_split_layer():
    # the ranks together index one L x H layer; the job takes its slowest rank's time
    assert bench.job_value(131072, 16, 50.0) == 131072 * 16 / 0.05
    assert bench.job_value(1024, 8, 2.0) == 1024 * 8 / 0.002


def test_clock_summary_flags_throttle_reasons():
    cs = bench.ClockSampler(0)

    class Done:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    cs.proc = Done()
    cs.lines = [
        "0, 1965, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1700, 1965, 995.0, 0x4, Not Active, Not Active, Not Active, Active",
        "garbage",
    ]
    s = cs.stop()
    assert s["sm_mhz"] == 1800 and s["sm_max_mhz"] == 1965 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]
