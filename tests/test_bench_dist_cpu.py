"""Host logic of the benchmark's multi-rank path, on CPU with gloo (2 ranks).

Every rank runs its own replica (weak scaling, no data-path collective); the
only collectives are the barrier and the max / sum of the per-rank timings,
which these tests check.  Also: argument parsing and the clock summary."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w, local = bench.dist_env()
    d = bench.dist_init(w, "gloo")
    try:
        dev = torch.device("cpu")
        ms = 10.0 + 5.0 * r                      # the slower rank decides
        mx = bench.max_over_ranks(ms, d, dev)
        tok = bench.sum_over_ranks(100.0 * (r + 1), d, dev)
        out[r] = (r, w, local, mx, tok)
    finally:
        d.barrier()
        d.destroy_process_group()


def test_two_rank_timing_reduction():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    for r, (rank, world, local, mx, tok) in res.items():
        assert (rank, world, local) == (r, 2, r)
        assert mx == 15.0                        # max over ranks
        assert tok == 300.0                      # whole-job units


def test_single_rank_needs_no_process_group(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    rank, world, local = bench.dist_env()
    assert (rank, world, local) == (0, 1, 0)
    assert bench.dist_init(world, "gloo") is None
    assert bench.max_over_ranks(3.5, None, None) == 3.5


def test_parse_args_defaults_and_guards():
    a = bench.parse_args([])
    assert a.gpus == 1 and a.warmup >= 3 and a.steps >= 1
    assert a.workload == "ffn_relu2_llama7b" and a.batch == 1
    assert bench.parse_args(["--workload", "prefill_bf16_2048"]).batch == 2048
    with pytest.raises(SystemExit):
        bench.parse_args(["--warmup", "2"])
    # the gate-first layer exists only for the dReLU FFN, and says so in its config
    with pytest.raises(SystemExit):
        bench.parse_args(["--gate-first"])
    g = bench.parse_args(["--workload", "ffn_drelu_mistral7b", "--gate-first", "--batch", "4"])
    assert g.gate_first and g.batch == 4
    assert "gate first" in bench.workload_desc(g, g.batch)
    assert "gate first" not in bench.workload_desc(bench.parse_args(["--workload", "ffn_drelu_mistral7b"]), 1)


def test_clock_summary():
    lines = [
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1950, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1965, 1965, 800.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage",
    ]
    s = bench.summarize_clocks(lines)
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]
    assert bench.summarize_clocks([])["samples"] == 0


def test_profile_digest_ignores_comments():
    """A profile stays valid across comment edits, not across code edits."""
    code = 'int f(int a) { // add one\n  return a + 1; /* done */ }\nconst char* s = "// not a comment";\n'
    same = 'int f(int a) {\n  return a + 1; }\n\n\nconst char* s = "// not a comment";  // note\n'
    other = 'int f(int a) {\n  return a + 2; }\nconst char* s = "// not a comment";\n'
    assert bench._code_only(code) == bench._code_only(same)
    assert bench._code_only(code) != bench._code_only(other)
    assert '"// not a comment"' in bench._code_only(code)


def test_profile_traffic_is_reported_only_for_the_current_kernel_code():
    """Every committed kernel profile records the digest of the code it was
    taken on; the bench line reports its DRAM traffic only while that digest
    matches the current kernel source (a changed kernel reads as null)."""
    import glob
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    names = [os.path.basename(p)[:-3] for p in glob.glob(os.path.join(root, "profiles", "*.md"))
             if os.path.basename(p).split("_")[0] in bench.KERNEL_SOURCES]
    assert names
    for name in names:
        vals = {}
        with open(os.path.join(root, "profiles", name + ".md")) as f:
            for ln in f:
                if ln.startswith("- ") and ":" in ln:
                    k, v = ln[2:].split(":", 1)
                    vals[k.strip()] = v.strip().strip("`")
        assert "source_digest" in vals and "dram_bytes_per_launch" in vals, name
        current = vals["source_digest"] == bench.kernel_source_digest(name)
        assert (bench.profiled_traffic(name) is not None) == current, name


def test_reference_arm_runs_the_oracle_on_the_same_workload():
    """`bench.py --impl reference` times the oracle on the host and prints the
    contract's line, with the same workload description as our arm."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                        "--workload", "linear_f32_512", "--steps", "5", "--warmup", "3",
                        "--ref-seconds", "1"], capture_output=True, text=True, timeout=300, cwd=root)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "tokens/s"
    assert line["metric"] == bench.METRIC and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    args = bench.parse_args(["--workload", "linear_f32_512"])
    assert line["config"]["workload"] == bench.workload_desc(args, args.batch)
    # both arms carry the same config keys
    ours = bench.run_config(bench.workload_desc(args, args.batch), args.batch, 1, 2, "l2", "p")
    assert set(line["config"]) == set(ours)
