"""Replica sharding across ranks (gloo, world size 2, CPU): each rank draws exactly
its slice of the global batch, and the timing reduction is the max over ranks."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_sparse_10_b200 import replicas, synth

WL = synth.Decode("tiny_decode", "hybrid", B=2, L=4096, H=16, m=4, k=64, win=16, m_hca=128)


def _wire(t):
    """Exact widening to a dtype gloo transports (bf16 -> fp32, uint8 -> int32)."""
    t = t.contiguous()
    if t.dtype == torch.bfloat16:
        return t.float()
    if t.dtype == torch.uint8:
        return t.to(torch.int32)
    return t


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = synth.decode_inputs(WL, seed=0, batch=replicas.shard(rank, WL.B))
        parts = {}
        for name in ("q", "kIc", "nope", "scale", "hca_rope"):
            t = _wire(x[name])
            gathered = [torch.empty_like(t) for _ in range(world)]
            dist.all_gather(gathered, t)
            parts[name] = torch.cat(gathered).numpy()
        mx = replicas.max_over_ranks(1.5 + rank)
        if rank == 0:
            np.savez(os.path.join(out_dir, "gathered.npz"), mx=mx, **parts)
    finally:
        dist.destroy_process_group()


def test_shards_concatenate_to_the_global_batch(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    got = np.load(tmp_path / "gathered.npz")
    assert float(got["mx"]) == 2.5
    full = synth.decode_inputs(synth.Decode("tiny_decode", "hybrid", B=WL.B * world, L=WL.L, H=WL.H, m=WL.m,
                                            k=WL.k, win=WL.win, m_hca=WL.m_hca), seed=0)
    for name in ("q", "kIc", "nope", "scale", "hca_rope"):
        assert np.array_equal(got[name], _wire(full[name]).numpy()), name


def test_shard_ranges():
    assert replicas.shard(0, 8) == slice(0, 8)
    assert replicas.shard(3, 8) == slice(24, 32)
    assert replicas.max_over_ranks(3.0) == 3.0
