"""Multi-rank plumbing of bench.py on CPU: two gloo ranks on 127.0.0.1.

The path shards by layer (each rank quantizes its own layer, no collective on
the data path); what crosses ranks is only the timing: a barrier and the
max-over-ranks of the device times.  These tests run those pieces with real
process groups, and check the reference arm's one-line JSON contract.
"""
import json
import os
import socket
import subprocess
import sys
from pathlib import Path

import pytest
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _load_bench():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", ROOT / "bench.py")
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, str(ROOT))
    bench = _load_bench()
    from awq_activation_aware_b200 import synth
    dist = bench.dist_init(world, "gloo")
    bench.barrier(world)
    mx = bench.reduce_max([float(rank + 1), 10.0 - rank, 3.5], world, "cpu")
    cfg = bench.rank_layer_config(synth.CONFIGS["attn4096"], rank)
    bench.barrier(world)
    dist.destroy_process_group()
    q.put((rank, mx, cfg.seed, cfg.N, cfg.K, cfg.T))


def test_two_gloo_ranks_max_and_layer_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, seed, N, K, T in res:
        assert mx == [2.0, 10.0, 3.5]           # element-wise max over ranks, same on every rank
        assert (N, K, T) == (4096, 4096, 4096)  # same shape on every rank (weak scaling)
    assert res[0][2] != res[1][2]               # but each rank has its own layer


def test_single_rank_reduce_is_identity():
    bench = _load_bench()
    assert bench.reduce_max([1.0, 2.0], 1, "cpu") == [1.0, 2.0]


def _run_reference(env_extra):
    env = dict(os.environ, **env_extra)
    cmd = [sys.executable, str(ROOT / "bench.py"), "--impl", "reference", "--config", "layer512",
           "--steps", "1", "--warmup", "0", "--cpu-rows", "16"]
    return subprocess.run(cmd, capture_output=True, text=True, env=env, timeout=600, cwd=ROOT)


def test_reference_arm_json_line():
    r = _run_reference({"WORLD_SIZE": "1", "RANK": "0"})
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["unit"] == "TFLOP/s" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_do_no_work():
    r = _run_reference({"WORLD_SIZE": "2", "RANK": "1"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


# ---------------------------------------------------------------------------
# One layer's rows split across ranks (awq_activation_aware_b200.sharded):
# the plumbing runs with two gloo ranks, with the library's kernels stood in
# for by the oracle on the CPU (each stand-in follows the C ABI's definition,
# awq_search_layer_part normalising by the layer's row count).
# ---------------------------------------------------------------------------
def _row_split_worker(rank, world, port, q, N, K, T, unit):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, str(ROOT))
    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle
    from awq_activation_aware_b200 import sharded, synth

    dist.init_process_group("gloo", rank=rank, world_size=world)
    W, X, _ = synth.generate(synth.make_config(N, K, T, seed=31, outlier_frac=0.03))
    r0, r1 = sharded.shard_rows(N, world, rank, unit=unit)

    def fake_stats(Xt):
        return torch.from_numpy(oracle.act_stats(Xt.numpy()))

    def fake_search(Wp, Xt, a, al, bits, group, workspace=None, zero_point=True, rows_total=None):
        r = oracle.search(Wp.numpy(), Xt.numpy(), a.numpy(), bits, group, al.numpy(), zero_point=zero_point)
        return torch.from_numpy((r["row_sums"].sum(axis=1) / (rows_total * Xt.shape[0])).astype(np.float32))

    def fake_pack(Wp, a, al, losses, bits, group, zero_point=True):
        pk = oracle.pack(Wp.numpy(), a.numpy(), bits, group, al.numpy(), losses.numpy().astype(np.float64),
                         zero_point=zero_point)
        return {"best_idx": torch.tensor([pk["best"]]), "codes": torch.from_numpy(pk["codes"])}

    sharded.act_stats, sharded.search_layer, sharded.pack = fake_stats, fake_search, fake_pack
    al = torch.from_numpy(synth.default_alphas())
    res = sharded.quantize_layer_rows(torch.from_numpy(np.ascontiguousarray(W[r0:r1])), torch.from_numpy(X), N,
                                      alphas=al)
    dist.destroy_process_group()
    q.put((rank, r0, r1, res["losses"].numpy().tolist(),
           int(res["best_idx"][0]) if "best_idx" in res else None,
           res["codes"].numpy() if "codes" in res else None))


@pytest.mark.parametrize("N,unit", [(200, 64), (200, 256)])
def test_row_split_two_ranks_matches_whole_layer(N, unit):
    """Two ranks: the all-reduced losses equal the whole layer's MSE, both
    ranks take the same argmin, and the parts' codes are the whole layer's
    rows.  With 256-row units the second rank holds no rows and still takes
    part in the all-reduce."""
    import numpy as np

    import oracle
    from awq_activation_aware_b200 import synth
    K, T = 256, 48
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_row_split_worker, args=(r, 2, port, q, N, K, T, unit)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    W, X, _ = synth.generate(synth.make_config(N, K, T, seed=31, outlier_frac=0.03))
    al = synth.default_alphas()
    a = oracle.act_stats(X)
    whole = oracle.search(W, X, a, 4, 128, al)
    full_pack = oracle.pack(W, a, 4, 128, al, whole["losses"])
    assert res[0][2] == res[1][1] and res[0][1] == 0 and res[1][2] == N
    for rank, r0, r1, losses, best, codes in res:
        np.testing.assert_allclose(losses, whole["losses"], rtol=1e-6)
        assert losses == res[0][3]                       # the same bits on every rank
        if r1 > r0:
            assert best == full_pack["best"]
            assert np.array_equal(codes, full_pack["codes"][r0:r1])
        else:
            assert codes is None
