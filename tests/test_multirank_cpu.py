"""Multi-rank plumbing of bench.py on CPU: two gloo ranks.

The layer does not shard: on N GPUs the bench runs N replicas, each with its
own seeded token batches, and no collective touches the data path.  What the
ranks do share is the timing: the job time is the max over ranks, and the
job's throughput counts the tokens of every rank.  These tests run that code
(bench.max_over_ranks, bench.job_tokens_per_s, bench.replica_input_seed) in
two processes over gloo, and check that a replica's layer output (computed
with the oracle) depends only on its own rank's inputs.
"""
import json
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _replica_output(rank):
    """Oracle layer output of one replica's first batch (small E)."""
    import moe_inputs as mi
    import oracle

    import bench
    cfg = mi.CONFIGS[0]
    inp = mi.make_layer(0, 2, layer=0, device="cpu", E=16)
    x = mi.gen_x(2, cfg.H, bench.replica_input_seed(0, rank, 0), "cpu", cfg.x_bf16)
    hidden = oracle.rmsnorm(x.numpy(), cfg.eps)
    wr = inp.w_router.view(torch.int16).numpy().view(np.uint16)
    out = oracle.moe_layer(hidden, wr, None if inp.bias is None else inp.bias.numpy(), 16, 4,
                           cfg.fmt, cfg.I, inp.experts.numpy())
    return np.asarray(out["out_f32"], np.float64)


def _rank_main(rank, port, outdir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "RANK": str(rank), "WORLD_SIZE": str(WORLD), "LOCAL_RANK": str(rank)})
    import sys
    sys.path.insert(0, ROOT)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ws, r, local = bench.dist_env()
        # rank-dependent times: rank 1 is the slower one in ms, rank 0 in e2e
        mine = [10.0 + 5.0 * rank, 30.0 - 7.0 * rank]
        got = bench.max_over_ranks(mine, torch.device("cpu"))
        seeds = [bench.replica_input_seed(1, rank, g) for g in range(4)]
        y = _replica_output(rank)
        # the one allowed exchange is the timing max; gather outputs only to
        # let the test compare them
        ys = [torch.zeros(y.shape, dtype=torch.float64) for _ in range(WORLD)]
        dist.all_gather(ys, torch.from_numpy(y))
        res = {"env": [ws, r, local], "max": got, "seeds": seeds,
               "y_all": [t.numpy().tolist() for t in ys]}
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def ranks(tmp_path_factory):
    out = tmp_path_factory.mktemp("ranks")
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, str(out))) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    for p in procs:
        if p.is_alive():
            p.kill()
            p.join()
    codes = [p.exitcode for p in procs]
    assert codes == [0] * WORLD, codes
    res = []
    for r in range(WORLD):
        with open(out / f"rank{r}.json") as f:
            res.append(json.load(f))
    return res


def test_env_is_read_per_rank(ranks):
    for r, res in enumerate(ranks):
        assert res["env"] == [WORLD, r, r]


def test_job_time_is_max_over_ranks(ranks):
    for res in ranks:
        assert res["max"] == [15.0, 30.0]


def test_replicas_draw_distinct_batches(ranks):
    a, b = ranks[0]["seeds"], ranks[1]["seeds"]
    assert len(set(a)) == len(a) and not set(a) & set(b)


def test_replica_output_depends_only_on_its_own_rank(ranks):
    y0 = np.asarray(ranks[0]["y_all"][0])
    y1 = np.asarray(ranks[0]["y_all"][1])
    assert not np.allclose(y0, y1)
    # each rank's output is reproduced by a lone process from that rank's seed
    np.testing.assert_array_equal(y0, _replica_output(0))
    np.testing.assert_array_equal(y1, _replica_output(1))
    # and both ranks saw the same gathered values
    np.testing.assert_array_equal(np.asarray(ranks[1]["y_all"]), np.asarray(ranks[0]["y_all"]))


def test_job_throughput_counts_every_rank():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    # 4 tokens/step/rank, 100 steps, 2 ranks, 50 ms -> 800 tokens / 0.05 s
    assert bench.job_tokens_per_s(4, 100, 2, 50.0) == pytest.approx(16000.0)
    assert bench.max_over_ranks([1.5, 2.5], torch.device("cpu")) == [1.5, 2.5]


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        config, tokens, layers, warmup, steps = 1, 0, 0, 3, 1
    assert bench.run_reference(A()) is None


def test_bench_lines_name_config_tokens_and_layers():
    """The bench's line list: config:T or config:T:layers; the default ends
    with the headline (config 1, T = 4) and every decode line streams more
    weight bytes per step than the 126 MB L2."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import moe_inputs as mi
    assert bench.parse_lines("2:8192,0:1:48,1:4") == [(2, 8192, None), (0, 1, 48), (1, 4, None)]
    lines = bench.parse_lines(bench.DEFAULT_LINES)
    assert lines[-1] == (1, 4, None)
    for config, T, L in lines:
        cfg = mi.CONFIGS[config]
        if T > 16:
            continue
        layers = L or cfg.layers
        # at least one expert per token per layer: k experts of the format's blob size
        per_step = layers * min(cfg.E, cfg.k * T) * mi.expert_bytes(cfg.fmt, cfg.H, cfg.I)
        assert per_step > bench.L2_BYTES, (config, T, layers, per_step)


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the oracle, on the host cores) prints one
    JSON line with the arm's keys; a one-layer C0 line keeps it to seconds."""
    import subprocess
    import sys
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3", "--lines", "0:1:1"],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    r = json.loads(lines[0])
    assert r["impl"] == "reference" and r["unit"] == "tokens/s" and r["higher_is_better"]
    assert r["value"] > 0 and r["steps"] == 1 and r["warmup"] == 3 and r["n_gpus"] == 1
    assert r["config"]["T"] == 1 and r["config"]["layers"] == 1
    cb = r["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == r["value"] and cb["cores"] >= 1
    assert cb["sample"]
    assert r["e2e"] == {"value": r["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert r["ms_per_step"] == pytest.approx(1e3 / r["value"], rel=1e-2)
