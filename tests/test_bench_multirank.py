"""Host logic of bench.py's multi-rank path on CPU: two gloo ranks, the
max-over-ranks step time, the whole-job throughput, the reference arm that
runs on rank 0 only, and the keys of the JSON line."""
import json
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_path):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    d = bench.Dist()
    d.init("gloo")
    d.barrier()
    t_local = 1.0 + 0.5 * rank                 # rank 1 is the slow one
    t_max = d.max(t_local)
    value = bench.throughput(1e9, d.world, 10, t_max)
    d.barrier()
    if d.rank == 0:
        with open(out_path, "w") as f:
            json.dump({"t_max": t_max, "value": value, "world": d.world}, f)
    d.close()


def test_two_gloo_ranks_take_the_max_time(tmp_path):
    out = str(tmp_path / "r0.json")
    mp.start_processes(_rank_main, args=(2, _free_port(), out), nprocs=2, join=True, start_method="spawn")
    r = json.load(open(out))
    assert r["world"] == 2
    assert r["t_max"] == pytest.approx(1.5)
    # whole-job GB/s: both ranks' bytes over the slowest rank's time
    assert r["value"] == pytest.approx(1e9 * 2 * 10 / 1.5 / 1e9)


def _retake_main(rank, world, port, out_path):
    """Rank 1's first clock record shows a thermal slowdown, rank 0's is clean:
    both ranks must take the timed region again, in lock step."""
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    d = bench.Dist()
    d.init("gloo")
    calls = []

    def sample_and_time():
        d.barrier()                               # the real timed region brackets itself with barriers
        calls.append(len(calls))
        bad = rank == 1 and len(calls) == 1
        return 1.0 + len(calls), {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0,
                                  "reasons": ["sw_thermal_slowdown"] if bad else []}
    t, clocks = bench.timed_with_retake(d, sample_and_time)
    t_max = d.max(t)                              # the next collective must pair up across ranks
    with open(out_path + ".%d" % rank, "w") as f:
        json.dump({"calls": len(calls), "t": t, "t_max": t_max, "retaken": clocks.get("retaken", False)}, f)
    d.close()


def test_retake_is_collective_when_one_rank_rejects(tmp_path):
    out = str(tmp_path / "retake")
    mp.start_processes(_retake_main, args=(2, _free_port(), out), nprocs=2, join=True, start_method="spawn")
    r = [json.load(open(out + ".%d" % j)) for j in range(2)]
    for x in r:
        assert x["calls"] == 2 and x["retaken"] is True
        assert x["t"] == pytest.approx(3.0) and x["t_max"] == pytest.approx(3.0)


def test_no_retake_when_clean():
    d = _FakeDist(0, 1)
    d.max = lambda x, device=None: x
    n = []
    t, c = bench.timed_with_retake(d, lambda: (n.append(1) or 2.0, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0,
                                                                   "reasons": []}))
    assert len(n) == 1 and t == 2.0 and "retaken" not in c


class _FakeDist:
    def __init__(self, rank, world):
        self.rank, self.world, self.pg = rank, world, False


def test_reference_arm_runs_on_rank0_only(capsys):
    ns = type("A", (), {"steps": 1, "warmup": 0, "gpus": 2})()
    assert bench.run_reference(ns, _FakeDist(1, 2)) == 0
    assert capsys.readouterr().out == ""          # a non-zero rank does no work and prints nothing


def test_json_line_carries_the_contract_keys():
    line = bench.assemble_line(value=1.0, unit="GB/s", n_gpus=2, steps=3, warmup=3, ms_per_step=1.0,
                               extra={"config": bench.config_dict()})
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config"):
        assert k in line
    assert line["scaling"] == "weak" and line["higher_is_better"] is True
    assert line["config"]["workload"] == bench.WORKLOAD


def test_clock_rejection_rule():
    ok = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    capped = {"sm_mhz": 1300.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    thermal = {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_thermal_slowdown"]}
    locked = {"sm_mhz": 1100.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert not bench.clocks_rejected(ok) and not bench.clocks_rejected(capped)
    assert bench.clocks_rejected(thermal) and bench.clocks_rejected(locked)
    assert not bench.clocks_rejected(None)


def test_clock_sampler_keeps_samples_inside_the_timed_region(tmp_path, monkeypatch):
    """nvidia-smi is replaced by a script: samples before begin() report a
    thermal slowdown, samples after it a power cap only."""
    flag = tmp_path / "timed"
    fake = tmp_path / "nvidia-smi"
    fake.write_text("#!/bin/sh\nwhile true; do\n"
                    "  if [ -e %s ]; then echo '1950, 1965, 100, 900.0, 0x0000000000000004';\n"
                    "  else echo '1200, 1965, 100, 900.0, 0x0000000000000020'; fi\n"
                    "  sleep 0.02\ndone\n" % flag)
    fake.chmod(0o755)
    monkeypatch.setenv("PATH", str(tmp_path) + os.pathsep + os.environ["PATH"])
    s = bench.ClockSampler(None, interval_ms=20)
    s.start()
    import time
    time.sleep(0.2)
    flag.write_text("")
    time.sleep(0.1)
    s.begin()
    time.sleep(0.4)
    s.end()
    c = s.stop()
    assert c["samples_in_timed_region"] >= 5
    assert c["sm_mhz"] == 1950.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"]
    assert not bench.clocks_rejected(c)


def _shard_bounds(n_out, world, rank):
    from residual_binarized_weight_b200.rbw import shard_bounds
    return shard_bounds(n_out, world, rank)


def _rowsplit_main(rank, world, port, out_path):
    """Each rank applies its row shard (oracle planes of its rows; the
    recurrence is row-local) and the shards are all-gathered along N."""
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import numpy as np
    import torch
    import oracle
    from residual_binarized_weight_b200 import synth
    d = bench.Dist()
    d.init("gloo")
    N, K, k, M = 300, 256, 2, 3                       # ragged: 10 row tiles over the ranks
    rng = np.random.default_rng(4)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k, iters=4)
    X = synth.activations(M, K, seed=2)
    r0, r1 = _shard_bounds(N, world, rank)
    planes, g16, h16, _, _ = oracle.pack(W[r0:r1], g[:, r0:r1], h, k)
    y_local = torch.from_numpy(oracle.apply(planes, g16, h16, r1 - r0, K, k, X))
    y = bench.rowsplit_gather(d, y_local, N, _shard_bounds)
    if rank == 0:
        planes, g16, h16, _, _ = oracle.pack(W, g, h, k)
        ref = oracle.apply(planes, g16, h16, N, K, k, X)
        np.save(out_path, np.stack([y.numpy(), ref]))
    d.close()


def test_row_split_all_gather_reassembles_the_full_output(tmp_path):
    out = str(tmp_path / "rs.npy")
    mp.start_processes(_rowsplit_main, args=(2, _free_port(), out), nprocs=2, join=True, start_method="spawn")
    import numpy as np
    y, ref = np.load(out)
    assert y.shape == ref.shape == (3, 300)
    assert np.array_equal(y, ref)                     # the same float64 oracle on every row


def test_shard_bounds_tile_aligned_and_complete():
    from residual_binarized_weight_b200.rbw import shard_bounds
    for n in (1, 31, 32, 300, 4096, 11008):
        for world in (1, 2, 3, 4, 8):
            b = [shard_bounds(n, world, r) for r in range(world)]
            assert b[0][0] == 0 and b[-1][1] == n
            for (a0, a1), (c0, c1) in zip(b, b[1:]):
                assert a1 == c0
            assert all(r0 % 32 == 0 and r0 <= r1 for r0, r1 in b)
