"""Two-rank (gloo, CPU) tests of the multi-GPU host path of bench.py.

The forward pass shards by independent problems: every rank runs its own
batch with no data-path collective, and the only collectives are the
measurement barrier and the max over ranks of the timed milliseconds.  These
tests run those pieces as two gloo ranks on the CPU:

- the max over ranks and the whole-job throughput;
- each rank's share of the global batch is distinct, and the shares together
  are the global batch;
- running the oracle rank by rank on the shares equals running it once on the
  global batch (the problems are independent, so sharding changes nothing);
- the reference arm does no work on ranks other than 0.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        sys.path.insert(0, ROOT)
        import bench
        import oracle as O
        import workloads as W

        # max over ranks and whole-job throughput
        ms = bench.max_over_ranks(1.5 + rank, world, "cpu")
        tflops = bench.whole_job_tflops(1e12, world, ms)

        # this rank's share of the global batch: tiny workload, one head
        w = W.with_overrides(W.BY_NAME["tiny_f32"], Hq=1, Hkv=1)
        b0 = bench.rank_batch0(rank, w.B)
        inp = W.make_inputs(w, batch0=b0)
        res = O.psa_head(inp.as_f64("q", 0, 0), inp.as_f64("k", 0, 0), inp.as_f64("v", 0, 0),
                         w.q_blk, w.kv_blk, W.thresholds(w), w.causal, w.forced_prefix_tokens)

        # head sharding of one problem: this rank's heads through the oracle
        wh = W.with_overrides(W.BY_NAME["tiny_f32"], Hq=4, Hkv=2, seed=3)
        hi = W.make_inputs(wh)
        import level_sparse_attention_b200 as PB
        q0, q1, kv0, kv1 = PB.head_shard(wh.Hq, wh.Hkv, rank, world)
        grp = wh.Hq // wh.Hkv
        shard_out = np.stack([
            O.psa_head(hi.as_f64("q", 0, h), hi.as_f64("k", 0, h // grp), hi.as_f64("v", 0, h // grp),
                       wh.q_blk, wh.kv_blk, W.thresholds(wh)).O for h in range(q0, q1)])
        assert all(kv0 <= h // grp < kv1 for h in range(q0, q1))

        # the reference arm returns without work on rank != 0
        class A:
            workload, steps, warmup, gpus = "tiny_f32", 1, 0, world
        ref = bench.run_reference(A, rank, world) if rank != 0 else None

        dist.barrier()
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), ms=ms, tflops=tflops, b0=b0,
                 q=inp.q, out=res.O, lse=res.lse, level_map=res.mask.level_map,
                 ref_none=ref is None, shard=np.array([q0, q1]), shard_out=shard_out)
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def rank_results(tmp_path_factory):
    out = tmp_path_factory.mktemp("ranks")
    mp.start_processes(_rank_main, args=(WORLD, _free_port(), str(out)), nprocs=WORLD,
                       join=True, start_method="spawn")
    return [dict(np.load(out / f"rank{r}.npz")) for r in range(WORLD)]


def test_max_over_ranks_and_whole_job_value(rank_results):
    for r in rank_results:
        assert float(r["ms"]) == 2.5                    # max of 1.5 and 2.5
        assert float(r["tflops"]) == pytest.approx(2 * 1e12 / 2.5e-3 / 1e12)


def test_shares_are_distinct_and_cover_the_global_batch(rank_results):
    import workloads as W
    assert [int(r["b0"]) for r in rank_results] == [0, 1]
    assert not np.array_equal(rank_results[0]["q"], rank_results[1]["q"])
    w = W.with_overrides(W.BY_NAME["tiny_f32"], Hq=1, Hkv=1, B=WORLD)
    whole = W.make_inputs(w)
    for r, res in enumerate(rank_results):
        np.testing.assert_array_equal(res["q"][0], whole.q[r])


def test_sharded_oracle_equals_global_batch(rank_results):
    import oracle as O
    import workloads as W
    w = W.with_overrides(W.BY_NAME["tiny_f32"], Hq=1, Hkv=1, B=WORLD)
    whole = W.make_inputs(w)
    for b, res in enumerate(rank_results):
        ref = O.psa_head(whole.as_f64("q", b, 0), whole.as_f64("k", b, 0), whole.as_f64("v", b, 0),
                         w.q_blk, w.kv_blk, W.thresholds(w), w.causal, w.forced_prefix_tokens)
        np.testing.assert_array_equal(res["level_map"], ref.mask.level_map)
        np.testing.assert_array_equal(res["out"], ref.O)
        np.testing.assert_array_equal(res["lse"], ref.lse)


def test_reference_arm_idles_off_rank_zero(rank_results):
    assert bool(rank_results[1]["ref_none"])


def test_head_shards_together_equal_the_whole_problem(rank_results):
    import oracle as O
    import workloads as W
    wh = W.with_overrides(W.BY_NAME["tiny_f32"], Hq=4, Hkv=2, seed=3)
    hi = W.make_inputs(wh)
    shards = sorted((tuple(r["shard"]), r["shard_out"]) for r in rank_results)
    assert [s[0] for s in shards] == [(0, 2), (2, 4)]
    got = np.concatenate([s[1] for s in shards])
    for h in range(wh.Hq):
        ref = O.psa_head(hi.as_f64("q", 0, h), hi.as_f64("k", 0, h // 2), hi.as_f64("v", 0, h // 2),
                         wh.q_blk, wh.kv_blk, W.thresholds(wh)).O
        np.testing.assert_array_equal(got[h], ref)


@pytest.mark.parametrize("Hq,Hkv,world", [(40, 40, 8), (12, 12, 5), (28, 4, 8), (28, 4, 4),
                                          (48, 48, 3), (4, 2, 4), (8, 1, 2), (8, 1, 8), (6, 3, 1)])
def test_head_shard_plan(Hq, Hkv, world):
    import level_sparse_attention_b200 as PB
    G = Hq // Hkv
    got = [PB.head_shard(Hq, Hkv, r, world) for r in range(world)]
    covered = []
    for q0, q1, kv0, kv1 in got:
        covered += list(range(q0, q1))
        if q1 > q0:
            # the shard's own grouping is the global one: local head i reads local
            # KV head i // ((q1 - q0) / (kv1 - kv0)), global head q0 + i reads (q0 + i) // G
            Gs = (q1 - q0) // (kv1 - kv0)
            assert (q1 - q0) % (kv1 - kv0) == 0
            assert all(kv0 + i // Gs == (q0 + i) // G for i in range(q1 - q0))
    assert covered == list(range(Hq))                       # disjoint, in order, complete
    sizes = [q1 - q0 for q0, q1, _, _ in got]
    assert max(sizes) - min(sizes) <= G                     # balanced to within a group


def test_head_shard_rejects_uneven_group_splits():
    import level_sparse_attention_b200 as PB
    with pytest.raises(ValueError):
        PB.head_shard(28, 4, 0, 6)                          # 6 ranks, 4 KV heads
    with pytest.raises(ValueError):
        PB.head_shard(8, 1, 0, 16)                          # more ranks than query heads
