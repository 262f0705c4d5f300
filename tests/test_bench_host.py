"""Host logic of the benchmark, on CPU.

Replicas: each rank drafts its own sequences with its own inputs; the only
cross-rank steps are the barrier, the slowest rank's device time and the
sum of verified tokens.  Two gloo ranks check that reduction and that
replicas draw distinct seeded inputs.  Also: the DRAM-traffic record is
honoured only for the sources it was captured on, and the accepted-length
statistics.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
import fm_synth as fs


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms, verified = bench.reduce_over_ranks(dist, "cpu", 1.5 + rank, 10.0 * (rank + 1), world)
        out.put((rank, ms, verified))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_reduce_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for rank, ms, verified in res:
        assert ms == pytest.approx(2.5)          # the slowest rank's time
        assert verified == pytest.approx(30.0)   # tokens of both replicas


def test_single_process_reduction():
    assert bench.reduce_over_ranks(None, "cpu", 3.0, 7.0, 1) == (3.0, 7.0)


def test_replicas_draw_distinct_rounds():
    seeds = {bench.round_seed(i, r) for r in range(8) for i in range(32)}
    assert len(seeds) == 8 * 32
    w = fs.WORKLOADS["tiny_f32"]
    a = fs.round_inputs(w, bench.round_seed(0, 0))
    b = fs.round_inputs(w, bench.round_seed(0, 1))
    assert not np.array_equal(a.noise, b.noise)
    assert not np.array_equal(a.u_draft, b.u_draft)


def test_stored_traffic_follows_the_sources(tmp_path):
    # a DRAM-traffic record counts only while the kernel sources are the
    # ones it was captured on
    import json
    rec = {"k": {"wl": {"dram_bytes_per_launch": 123, "source_sha1": bench.source_sha1()}}}
    p = tmp_path / "t.txt"
    p.write_text(json.dumps(rec))
    assert bench.stored_traffic("k", "wl", str(p)) == 123
    assert bench.stored_traffic("k", "other", str(p)) is None
    rec["k"]["wl"]["source_sha1"] = "0" * 40
    p.write_text(json.dumps(rec))
    assert bench.stored_traffic("k", "wl", str(p)) is None


def test_acceptance_stats():
    st = bench.acceptance_stats([[0, 3], [16, 3]], 16)
    assert st["mean"] == pytest.approx(5.5)
    assert st["hist"][0] == 1 and st["hist"][3] == 2 and st["hist"][16] == 1
    assert sum(st["hist"]) == 4
    assert st["p_reach"][0] == 0.75      # three of four reach position 1
    assert st["p_reach"][3] == 0.25      # only the full block passes position 4
    assert st["p_reach"][15] == 0.25


def test_source_hash_ignores_comments_only():
    src = 'const char* s = "a // b"; // note\n/* block */ int x = 1;  \n\n'
    assert bench._strip_comments(src) == 'const char* s = "a // b";\n int x = 1;'
    assert bench._strip_comments("int y = '\\''; // c") == "int y = '\\'';"


def _env_rank_main(out_dir):
    # a rank started by bench.launch_local: everything comes from the
    # environment, as under torchrun
    import datetime

    import torch
    import torch.distributed as dist
    rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    assert os.environ["MASTER_ADDR"] == "127.0.0.1"
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        ms, verified = bench.reduce_over_ranks(dist, "cpu", 2.0 * (rank + 1), 5.0, world)
        t = torch.tensor([float(rank)])
        dist.all_reduce(t)
        with open(os.path.join(out_dir, f"r{rank}"), "w") as f:
            f.write(f"{world} {int(os.environ['LOCAL_RANK'])} {ms} {verified} {t.item()}")
        dist.barrier()
    finally:
        dist.destroy_process_group()
    return 0


def _failing_rank():
    return 3 if os.environ["RANK"] == "1" else 0


def test_self_launch_two_gloo_ranks(tmp_path):
    # `bench.py --gpus N` without torchrun starts its N ranks itself
    bench.launch_local(2, _env_rank_main, str(tmp_path), timeout_s=180)
    for r in range(2):
        world, local, ms, verified, s = (tmp_path / f"r{r}").read_text().split()
        assert (int(world), int(local)) == (2, r)
        assert float(ms) == pytest.approx(4.0) and float(verified) == pytest.approx(10.0)
        assert float(s) == pytest.approx(1.0)


def test_self_launch_reports_a_failed_rank():
    with pytest.raises(RuntimeError):
        bench.launch_local(2, _failing_rank, timeout_s=120)


def test_8b_bs1_step_bytes_match_the_survey_count():
    # the concurrency-1 8B round moves ~1.999 GB: E, W_lm, block weights,
    # fc, context keys/values, noise and target logits; the key/value
    # weights of the round's new context rows are the QKV weights the
    # persistent pass streams anyway and are not counted twice
    w = fs.WORKLOADS["qwen3_8b_bs1"]
    ab = bench.algorithmic_bytes(w)
    total = sum(ab[k] for k in ("embed", "lm_head", "dit_gemm", "attn", "context", "verify"))
    assert bench.persistent_pass(w)
    assert total == pytest.approx(1.999e9, rel=2e-3)
    w5 = fs.WORKLOADS["qwen3_8b_bs64"]
    assert not bench.persistent_pass(w5)
    d = w5.shape.d
    assert bench.algorithmic_bytes(w5)["context"] > 6 * 2 * d * d * 2   # separate K/V projection


def test_clock_samples_of_the_timed_region():
    # samples are (before, after, MHz, reason bits); those overlapping the
    # region [10, 11] count, including one NVML call that spans all of it
    R = bench.ClockSampler.REASONS
    raw = [(9.0, 9.5, 1000, 0x0),        # before the region
           (9.9, 10.1, 1965, 0x4),       # overlaps its start: sw_power_cap
           (10.4, 10.5, 1965, 0x0),      # inside
           (10.9, 11.2, 1900, 0x8),      # overlaps its end: hw_slowdown
           (11.5, 11.6, 500, 0x20)]      # after
    mhz, names = bench.window_samples(raw, 10.0, 11.0, R)
    assert mhz == [1965, 1965, 1900]
    assert names == {"sw_power_cap", "hw_slowdown"}
    mhz, names = bench.window_samples([(9.0, 12.0, 1965, 0x0)], 10.0, 11.0, R)
    assert mhz == [1965] and names == set()
    assert bench.window_samples([], 10.0, 11.0, R) == ([], set())


def test_clock_summary_of_a_sampler():
    # the summary the bench line carries, without NVML: a sampler that
    # could not start reports why; one with samples reports their median
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c.ok, c.err = False, "no NVML"
    assert c.summary()["reasons"] == ["nvml unavailable: no NVML"]
    c.ok, c.max_mhz, c.window = True, 1965, 0.05
    c.samples, c.reasons = [1965, 1900, 1965], {"sw_power_cap"}
    s = c.summary()
    assert s["sm_mhz"] == 1965 and s["samples"] == 3 and s["reasons"] == ["sw_power_cap"]
    assert s["window_ms"] == 50.0 and s["sm_max_mhz"] == 1965
