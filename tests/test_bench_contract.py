"""bench.py's reference arm (the float64 oracle on the host cores) prints one JSON
line with the contract's keys; it needs no GPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "csa_prefill_t2048", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "tokens/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"]


def test_gpus_flag_must_match_the_launched_ranks():
    """--gpus N under a launcher that started a different number of ranks is refused (exit 2), before any GPU
    work, so a one-rank run can never be labelled as N GPUs."""
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert r.returncode == 2, (r.returncode, r.stderr[-2000:])
    assert "--gpus 2" in r.stderr
    assert not [ln for ln in r.stdout.splitlines() if ln.startswith("{")]


def test_prefill_timing_rotates_past_l2():
    """Prefill workloads whose per-step inputs and outputs fit in the 126 MB L2 are timed over a rotation of
    copies whose total exceeds it; larger ones use a single set.  The reference arm describes the same."""
    sys.path.insert(0, ROOT)
    import bench
    from long_context_sparse_10_b200 import synth
    for name in ("csa_prefill_t2048", "hca_prefill_t8192"):
        wl = synth.WORKLOADS[name]
        run = bench.PrefillRun.__new__(bench.PrefillRun)  # host inputs only, no GPU
        run.wl, run.host, run.csa_kind = wl, synth.prefill_inputs(wl, seed=0), wl.kind == "csa"
        set_bytes, nsets = run.rotation()
        host = sum(v.numel() * v.element_size() for v in run.host.values())
        assert set_bytes == host + wl.B * wl.T * wl.H * (128 * 2 + 4)
        assert nsets * set_bytes > 126e6 and (nsets == 1 or (nsets - 1) * set_bytes < 1.5 * 126e6)
        l2 = run.describe(1)["l2"]
        assert ("rotate" in l2) == (nsets > 1), l2


def test_decode_description_states_graph_steps_and_hca_budget():
    """The decode line names how many whole steps one graph launch holds and, for the hybrid step with bf16
    indexer keys, the SM budget of its HCA branch (the E4M3 / E2M1 steps keep every SM for it)."""
    sys.path.insert(0, ROOT)
    import bench
    from long_context_sparse_10_b200 import synth
    expect = {"hybrid_decode_l1m": 80, "hybrid_decode_l1m_fp8idx": 0, "hybrid_decode_l1m_fp4idx": 0,
              "csa_decode_l131072": 0}
    for name, sms in expect.items():
        wl = synth.WORKLOADS[name]
        assert bench.DecodeRun.hca_sms_for(wl) == sms, name
        run = bench.DecodeRun.__new__(bench.DecodeRun)  # no GPU
        run.wl, run.hybrid = wl, wl.kind == "hybrid"
        cfg = run.describe(1)
        assert cfg["timing"] == f"CUDA graph replay, {bench.DecodeRun.graph_steps} whole steps captured per launch"
        assert ("held to 80 SMs" in cfg["workload"]) == (sms == 80), cfg["workload"]
