"""Head-parallel split of one layer (long_context_sparse_stripe_b200.shard) on the host: two gloo
ranks each take the KV heads g with g mod 2 = rank and their query heads, build the indices and
the attention of their shard with the CPU oracle, and assemble O with one all-gather. Every head
is covered exactly once, each rank's index arrays equal the single-process ones of its heads bit
for bit, and the gathered output equals the single-process output (each head's work reads only
its own queries and its KV head's keys and values, so the split changes nothing)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import gen  # noqa: E402
from long_context_sparse_stripe_b200 import shard  # noqa: E402

CASES = {
    # Four KV heads over two ranks (two each), GQA of two.
    "even": gen.Workload("shard-even", batch=1, n_q_heads=8, n_kv_heads=4, seq_len=1024,
                         head_dim=64, segment_len=256, block_size=64, tau=0.005, seed=41,
                         amp=12.0, stripe_frac=0.05, q_shift=3.0),
    # Three KV heads over two ranks (two and one: the gather pads the smaller shard), one key
    # ordering per KV head, two batch elements.
    "uneven": gen.Workload("shard-uneven", batch=2, n_q_heads=6, n_kv_heads=3, seq_len=1024,
                           head_dim=64, segment_len=256, block_size=64, tau=0.005, seed=42,
                           amp=12.0, stripe_frac=0.05, q_shift=3.0, shared_key_order=1),
}
NAMES = ("perm_q", "perm_k", "sel_cnt", "sel_blk", "local_tiles")


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def rank_main(rank, world, port, case, out_dir):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    from datetime import timedelta

    import oracle
    dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    w = CASES[case]
    q, k, v = gen.make_inputs(w)
    sub = shard.shard_config(w, rank, world)
    qs, ks, vs = shard.shard_inputs(q, k, v, rank, world)
    ocfg = oracle.config(sub)
    idx = oracle.build_indices(ocfg, qs, ks, n_threads=2)
    out, _ = oracle.attention(ocfg, qs, ks, vs, idx, n_threads=2)
    o_shard = torch.from_numpy(out).reshape(w.batch, sub.n_q_heads, w.seq_len, w.head_dim)
    full = shard.gather_output(o_shard, w.n_q_heads, w.n_kv_heads, rank, world, dist)
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), full=full.numpy(),
             heads=np.array(shard.query_heads(w.n_q_heads, w.n_kv_heads, rank, world)),
             **{n: idx[n] for n in NAMES})
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("case", sorted(CASES))
def test_kv_head_split_over_two_gloo_ranks(tmp_path, case):
    import oracle
    world = 2
    mp.spawn(rank_main, args=(world, free_port(), case, str(tmp_path)), nprocs=world, join=True)
    w = CASES[case]
    q, k, v = gen.make_inputs(w)
    ocfg = oracle.config(w)
    ref = oracle.build_indices(ocfg, q, k)
    want, _ = oracle.attention(ocfg, q, k, v, ref)
    want = want.reshape(w.batch, w.n_q_heads, w.seq_len, w.head_dim)
    got = [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]
    heads = np.concatenate([g["heads"] for g in got])
    assert sorted(heads.tolist()) == list(range(w.n_q_heads))  # every head exactly once
    for g in got:
        h = g["heads"]
        for name in NAMES:
            np.testing.assert_array_equal(g[name], ref[name][:, h], err_msg=name)
        np.testing.assert_array_equal(g["full"], want)


def test_head_sets():
    assert shard.kv_heads(8, 1, 3) == [1, 4, 7]
    assert shard.query_heads(32, 8, 0, 2) == [0, 1, 2, 3, 8, 9, 10, 11, 16, 17, 18, 19,
                                              24, 25, 26, 27]
    cover = sorted(h for r in range(4) for h in shard.query_heads(32, 8, r, 4))
    assert cover == list(range(32))
    with pytest.raises(ValueError):
        shard.shard_config(gen.workload("llama-32k"), 15, 16)  # KV heads 0..7 only
