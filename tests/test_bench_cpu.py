"""Host-side checks of bench.py that need no GPU: the reference arm (the CPU oracle timed on the
host) prints exactly one JSON line with the contract's keys, a non-zero rank of it prints nothing,
the DRAM-traffic and pipe-counter records are reported only for the workload and code they were
captured on (comments aside), the reference arm's steps are what it ran, the fp32 work counts split by pair class,
the peaks file falls back when absent, and the algorithmic byte counts split into the parts that
grow with the instance count and the parts that do not."""
import importlib.util
import json
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CONTRACT = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
            "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config")


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _reference(extra_env=None):
    env = dict(os.environ, **(extra_env or {}))
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "1",
                           "--steps", "1", "--warmup", "0"], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_one_contract_line():
    r = _reference()
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in CONTRACT + ("impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["unit"] == "Mpix/s" and d["value"] > 0
    assert d["higher_is_better"] is True and d["data"] == "synthetic"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "Mpix/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == _bench().WORKLOADS[1]


def test_reference_arm_other_ranks_do_no_work():
    r = _reference({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def _copy_sources(tmp_path, srcs):
    for f in srcs:
        (tmp_path / f).parent.mkdir(parents=True, exist_ok=True)
        shutil.copy(os.path.join(ROOT, f), tmp_path / f)


def test_traffic_record_follows_workload_and_code(tmp_path, monkeypatch):
    """A record answers only for its workload and only while its sources' code is unchanged:
    rewording a comment keeps it, changing one token of code retires it."""
    b = _bench()
    srcs = ["gaussian_splatting_raster_b200/csrc/traverse.cuh",
            "gaussian_splatting_raster_b200/csrc/raster.cu"]
    _copy_sources(tmp_path, srcs)
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    rec = {"kernels": {"replay": {"workload": "w1", "dram_read_bytes": 300, "dram_write_bytes": 45,
                                  "sources": srcs, "code_sha256": b.code_digest(srcs)}}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "dram_traffic.json").write_text(json.dumps(rec))
    assert b.recorded_traffic("replay", "w1") == 345
    assert b.recorded_traffic("replay", "w2") is None
    assert b.recorded_traffic("render", "w1") is None
    f0 = tmp_path / srcs[0]
    text = f0.read_text()
    f0.write_text("// a reworded note\n/* and a block\n   comment */\n" + text + "\n\n")
    assert b.recorded_traffic("replay", "w1") == 345
    f0.write_text(text.replace("kAlphaMin = 1.0f / 255.0f", "kAlphaMin = 1.0f / 256.0f", 1))
    assert b.recorded_traffic("replay", "w1") is None


def test_pipe_record_follows_workload_and_code(tmp_path, monkeypatch):
    b = _bench()
    srcs = ["gaussian_splatting_raster_b200/csrc/raster.cu"]
    _copy_sources(tmp_path, srcs)
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    rec = {"kernels": {"render": {"workload": "w1", "fma_pipe_pct": 41.5, "alu_pipe_pct": 30.0,
                                  "issue_active_pct": 80.0, "sources": srcs,
                                  "code_sha256": b.code_digest(srcs)}}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "pipe_counters.json").write_text(json.dumps(rec))
    assert b.recorded_pipes("render", "w1") == {"fma_pipe_pct": 41.5, "alu_pipe_pct": 30.0,
                                                "issue_active_pct": 80.0}
    assert b.recorded_pipes("render", "w2") is None and b.recorded_pipes("replay", "w1") is None
    with open(tmp_path / srcs[0], "a") as fh:
        fh.write("static int extra;\n")
    assert b.recorded_pipes("render", "w1") is None


def test_code_text_drops_comments_only():
    b = _bench()
    src = ('int a = 1; // note\n/* block\n   x */ const char* s = "// kept"; char q = \'/\';\n'
           '\n#define X 1 /* y */\nfloat f = 2.0f;   \n')
    assert b.code_text(src) == ('int a = 1;\n  const char* s = "// kept"; char q = \'/\';\n'
                                '#define X 1\nfloat f = 2.0f;')
    # an escaped quote does not end a literal; a comment marker after it is still literal text
    src = 'printf("a\\"// b"); // c\nchar e = \'\\\'\'; /* d */ int z;\n'
    assert b.code_text(src) == 'printf("a\\"// b");\nchar e = \'\\\'\';   int z;'


def test_alu_work_counts_by_pair_class():
    """Every traversed pair costs the exponent and skip decision; only composited pairs cost
    alpha and the pass's own arithmetic."""
    b = _bench()
    for k, (a, c) in b.ALU_OPS.items():
        assert b.alu_ops(k, 1, 0) == a and b.alu_ops(k, 0, 1) == c
        assert b.alu_ops(k, 1000, 10) == 1000 * a + 10 * c
    # alpha (15) is part of every pass's composited cost; the replay does the most per pair;
    # only the render (and the passes that still visit their warps' union entries) decide
    # traversed pairs
    assert min(c for _, c in b.ALU_OPS.values()) >= 15 + 10
    assert b.ALU_OPS["replay"][1] > b.ALU_OPS["render"][1]
    assert b.ALU_OPS["render"][0] > 0 and b.ALU_OPS["replay"][0] == 0


def test_reference_steps_are_what_ran():
    """The reference arm's steps x ms_per_step is time it actually spent (no extrapolated
    samples): it fits inside the process's own wall time."""
    import time
    t0 = time.perf_counter()
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "2",
                        "--steps", "2", "--warmup", "1"], cwd=ROOT, capture_output=True,
                       text=True, timeout=600)
    wall = time.perf_counter() - t0
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads(r.stdout.strip())
    assert d["steps"] == 2 and "whole" in d["cpu_baseline"]["sample"]
    assert d["steps"] * d["ms_per_step"] * 1e-3 < wall
    # one step is one 128 x 128 view: value and ms_per_step describe the same time
    assert abs(d["value"] - 128 * 128 / (d["ms_per_step"] * 1e3)) < 1e-6 * d["value"]


def test_peaks_file_and_fallback(tmp_path, monkeypatch):
    b = _bench()
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    assert b.load_peaks()["source"] == "fallback"
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 1234.5, "sm_max_mhz": 1900}))
    assert b.load_peaks() == {"hbm_gbs": 1234.5, "sm_max_mhz": 1900.0, "source": "measured"}


def test_algorithmic_bytes_split_by_what_they_scale_with():
    b = _bench()
    sys.path.insert(0, ROOT)
    from synth import scenes
    sc = scenes.make(2)
    a = b.algorithmic_bytes(sc, 1000, 0)
    a2 = b.algorithmic_bytes(sc, 2000, 0)
    per_instance = {"emit": 8, "tile_hist": 4, "tile_scatter": 12, "render": 40, "replay": 40,
                    "backward": 40, "features": 40, "scatter": 80, "render_replay": 80}
    for k, v in a.items():
        assert v >= 0, k
        assert a2[k] - v == 1000 * per_instance.get(k, 0), k
    # one depth pass more adds one histogram read and one key+index read and write per (v, g)
    a4 = b.algorithmic_bytes(sc, 1000, 0, depth_passes=4)
    VG = sc.V * sc.G
    assert a4["depth_hist"] - a["depth_hist"] == 4 * VG
    assert a4["depth_scatter"] - a["depth_scatter"] == 16 * VG


def test_parity_report_locates_differences():
    """The whole-view comparison the bench prints: identical outputs give zero errors; a token
    block or a pixel changed on one side shows up in that block's and that output's figures."""
    import numpy as np
    b = _bench()
    rng = np.random.default_rng(3)
    d, G, H, W = 4, 500, 8, 16
    K = 9 + 3 * d
    zo = rng.normal(size=(G, K))
    zo[:, 4 + 3 * d] = np.log(rng.uniform(1e-5, 2.0, G))  # log q_g: some below 1e-3
    o = {"img": rng.uniform(size=(1, H, W, 3)), "T": rng.uniform(size=(1, H, W)),
         "n_contrib": rng.integers(0, 9, (1, H, W)).astype(np.int32), "tokens": zo}
    g = {"img": o["img"].astype(np.float32), "T": o["T"].astype(np.float32),
         "n_contrib": o["n_contrib"].copy(), "tokens": zo.astype(np.float32)}
    r = b.parity_report(g, o, d, chunk=64)
    assert r["T_final_mismatches"] == 0 and r["n_contrib_mismatches"] == 0
    assert r["colour_max_abs_err"] < 1e-7 and r["token_rel_err_max"] < 1e-6
    assert r["frac_pass_all"] == 1.0 and r["frac_pass_qg_ge_1e-3"] == 1.0
    assert r["gaussians_qg_ge_1e-3"] == int((np.exp(zo[:, 4 + 3 * d]) >= 1e-3).sum())
    assert set(r["token_block_rel_err_max"]) == {"b_mu", "s_alpha", "s_sh", "log_q", "eig",
                                                 "log_tr"}
    # one Gaussian's SH block off by 1 %, one pixel's colour by 1e-4, one count and one T changed
    g["tokens"][7, 4:4 + 3 * d] *= 1.01
    g["img"][0, 2, 3, 1] += 1e-4
    g["n_contrib"][0, 1, 1] += 1
    g["T"][0, 5, 5] = np.nextafter(g["T"][0, 5, 5], np.float32(2))
    r = b.parity_report(g, o, d, chunk=64)
    assert r["T_final_mismatches"] == 1 and r["n_contrib_mismatches"] == 1
    assert 0.9e-4 < r["colour_max_abs_err"] < 1.1e-4
    blk = r["token_block_rel_err_max"]
    assert 0.9e-2 < blk["s_sh"] < 1.1e-2
    assert all(v < 1e-6 for k, v in blk.items() if k != "s_sh")
    assert r["frac_pass_all"] == (G - 1) / G
    assert r["token_rel_err_max"] > 1e-4


def test_oracle_view_outputs_feed_the_report():
    """cpu_oracle_view(keep_outputs=True) hands back the arrays parity_report reads, shaped as the
    CUDA path's outputs of one view (compared here with themselves, rounded to fp32)."""
    import numpy as np
    b = _bench()
    sys.path.insert(0, ROOT)
    from synth import scenes
    sc = scenes.make(2)
    obs = np.random.default_rng(0).uniform(0, 1, (sc.V, sc.H, sc.W, 3)).astype(np.float32)
    s = b.cpu_oracle_view(sc, obs, keep_outputs=True)
    o = s["outputs"]
    assert o["img"].shape == (1, sc.H, sc.W, 3) and o["T"].shape == (1, sc.H, sc.W)
    assert o["n_contrib"].shape == (1, sc.H, sc.W)
    assert o["tokens"].shape == (sc.G, 9 + 3 * sc.d)
    g = {"img": o["img"].astype(np.float32), "T": np.asarray(o["T"]).astype(np.float32),
         "n_contrib": o["n_contrib"].astype(np.int32), "tokens": o["tokens"].astype(np.float32)}
    r = b.parity_report(g, o, sc.d)
    assert r["pixels"] == sc.H * sc.W and r["gaussians"] == sc.G
    assert r["T_final_mismatches"] == 0 and r["n_contrib_mismatches"] == 0
    assert r["token_rel_err_max"] < 1e-6 and r["frac_pass_all"] == 1.0
    assert b.cpu_oracle_view(sc, obs)["outputs"] is None


def test_no_collective_under_a_rank_branch():
    """Every rank must take the same collective steps: no reduction or barrier of bench.py sits
    inside a branch taken by some ranks only (a test of `rank`), where the other ranks would wait
    for it forever."""
    import ast
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    collectives = {"max_over_ranks", "pairs_sum_over_ranks", "barrier", "all_reduce",
                   "all_gather", "reduce_scatter_tensor", "broadcast"}

    def names(node):
        return {n.id for n in ast.walk(node) if isinstance(n, ast.Name)}

    bad = []
    for node in ast.walk(tree):
        if isinstance(node, (ast.If, ast.IfExp)) and "rank" in names(node.test):
            for sub in ast.walk(node):
                if isinstance(sub, ast.Call):
                    f = sub.func
                    name = f.id if isinstance(f, ast.Name) else getattr(f, "attr", None)
                    if name in collectives:
                        bad.append((sub.lineno, name))
    assert not bad, bad


def test_clock_samples_are_those_of_the_timed_region():
    b = _bench()
    S = b.ClockSampler
    idle, busy = "1200, 1965, 90.5, Not Active, Not Active, Not Active, Not Active", \
        "1965, 1965, 700.0, Not Active, Not Active, Not Active, Active"
    lines = [(0.0, idle), (1.0, idle), (2.0, busy), (2.1, busy), (2.2, "garbage"),
             (2.3, busy.replace("1965, 1965", "1905, 1965")), (5.0, idle)]
    r = S.summarize(lines, 1.5, 2.5)
    assert r["samples"] == 3 and r["window"] == "timed region"
    assert r["sm_mhz"] == 1965.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]
    # a region shorter than the interval: the first sample after its start stands for it
    r = S.summarize(lines, 2.35, 2.4)
    assert r["samples"] == 1 and r["sm_mhz"] == 1200.0 and r["window"].startswith("first")
    assert S.summarize(lines, 9.0, 9.5)["window"] == "no sample"


def test_clock_sampler_reads_a_live_sampler(tmp_path, monkeypatch):
    """The sampler against a stand-in nvidia-smi that prints one CSV sample every 20 ms: start()
    returns once a sample has arrived, and stop() keeps only the samples of the marked region."""
    import time
    b = _bench()
    fake = tmp_path / "nvidia-smi"
    fake.write_text("#!" + sys.executable + "\n"
                    "import sys, time\n"
                    "while True:\n"
                    "    print('1965, 1965, 500, Not Active, Not Active, Not Active, Active',"
                    " flush=True)\n"
                    "    time.sleep(0.02)\n")
    fake.chmod(0o755)
    monkeypatch.setenv("PATH", str(tmp_path) + os.pathsep + os.environ["PATH"])
    s = b.ClockSampler(None)
    t = time.monotonic()
    s.start()
    assert s.lines and time.monotonic() - t < 5
    s.mark()
    time.sleep(0.3)
    r = s.stop()
    assert r["window"] == "timed region" and r["samples"] >= 2
    assert r["sm_mhz"] == 1965.0 and r["reasons"] == ["sw_power_cap"]
    assert s.proc.poll() is not None  # the sampler process has ended


def test_parity_report_sign_and_cosine():
    """The experiment plan's score-check metrics in the report: identical tokens agree in sign
    everywhere and every block's cosine is 1; one flipped entry of one Gaussian's SH block lowers
    the sign agreement by one entry and that block's cosine only."""
    import numpy as np
    b = _bench()
    rng = np.random.default_rng(4)
    d, G = 9, 300
    K = 9 + 3 * d
    zo = rng.normal(size=(G, K))
    zo[:, 4 + 3 * d] = np.log(2.0)  # q_g = 2: every Gaussian counts
    o = {"img": np.zeros((1, 4, 4, 3)), "T": np.ones((1, 4, 4)),
         "n_contrib": np.zeros((1, 4, 4), np.int32), "tokens": zo}
    g = {"img": np.zeros((1, 4, 4, 3), np.float32), "T": np.ones((1, 4, 4), np.float32),
         "n_contrib": np.zeros((1, 4, 4), np.int32), "tokens": zo.copy()}
    r = b.parity_report(g, o, d, chunk=50)
    assert r["sign_agreement_qg_ge_1e-3"] == 1.0
    assert all(abs(c - 1) < 1e-12 for c in r["block_cosine_min_qg_ge_1e-3"].values())
    n_big = int((np.abs(zo) > 1e-4 * np.linalg.norm(zo, axis=1)[:, None]).sum())
    g["tokens"][11, 4 + 5] *= -1.0
    r = b.parity_report(g, o, d, chunk=50)
    assert r["sign_agreement_qg_ge_1e-3"] == (n_big - 1) / n_big
    cmin = r["block_cosine_min_qg_ge_1e-3"]
    assert cmin["s_sh"] < 1 - 1e-6
    assert all(abs(c - 1) < 1e-12 for k, c in cmin.items() if k != "s_sh")
    assert abs(r["block_cosine_median_qg_ge_1e-3"]["s_sh"] - 1) < 1e-12
