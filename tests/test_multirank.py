"""The multi-rank plumbing of bench.py on CPU: two gloo ranks.

The path shards with no exchange (segments and kv heads are independent),
so a multi-GPU run is N replicas, one batch of the same shape per rank.
What the ranks share is the timing: the job's time is the max over ranks,
and rank 0 alone prints.  The reference arm runs on rank 0 only."""
import json
import os
import socket

import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank's own step times: the job takes the slowest
        local = [3.0, 5.5][rank]
        job = bench.max_over_ranks(local, dist, "cpu")
        # each rank draws its own batch of the same shape
        lay = W.layout("decode_tinyllama_b64", seed=bench.rank_seed("decode_tinyllama_b64", rank))
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"job": job, "seq_lens": lay.seq_lens.tolist(), "num_tokens": lay.num_tokens}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time_and_draw_their_own_batches(tmp_path):
    port = _free_port()
    mp.spawn(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    r = [json.load(open(tmp_path / f"rank{i}.json")) for i in range(2)]
    assert r[0]["job"] == r[1]["job"] == 5.5
    assert r[0]["num_tokens"] == r[1]["num_tokens"] == 64          # same shape
    assert r[0]["seq_lens"] != r[1]["seq_lens"]                    # different draws


def test_one_rank_keeps_its_own_time():
    assert bench.max_over_ranks(7.25, None, "cpu") == 7.25


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    # ranks other than 0 exit at once, print nothing and do no work
    monkeypatch.setenv("RANK", "1")

    class Args:
        workload = "tiny_mixed"
        steps = 1
        warmup = 3
        gpus = 2

    assert bench.run_reference(Args()) == 0
    assert capsys.readouterr().out == ""


def test_rank_seeds_are_distinct_and_rank_zero_uses_the_workload_seed():
    seeds = [bench.rank_seed("mixed_qwen25_1p5b_t8192", r) for r in range(8)]
    assert seeds[0] == W.WORKLOADS["mixed_qwen25_1p5b_t8192"][1]
    assert len(set(seeds)) == 8
