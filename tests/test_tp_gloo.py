"""Tensor parallelism on CPU: two gloo ranks run the layout of
transformer_layer_residual_b200.tp with the oracle and check that the sharded
computation equals the unsharded one.

Rank r holds the K slice of the row-parallel output projection and computes its
partial output; the partials are gathered over gloo and summed by the oracle's
all-reduce (the sum fnl_tp_allreduce forms on the GPU); each rank then runs the
fused QKV op on its own heads and the gate/up op on its own rows. Rank 0 checks
the union of the shards against the single-rank computation.
"""
import os
import socket
import sys

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import oracle
    from transformer_layer_residual_b200 import tp
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    rng = np.random.default_rng(2024)   # the same draws on every rank
    M, Ko, K, Hq, Hkv, D, I, eps = 6, 32, 48, 4, 2, 8, 12, 1e-5
    bf = oracle.bf16_round
    a = bf(rng.normal(size=(M, Ko)))
    Wo = bf(rng.normal(0, Ko ** -0.5, (K, Ko)))
    resid = bf(rng.normal(size=(M, K)))
    gamma = bf(1 + 0.1 * rng.normal(size=K))
    Wqkv = bf(rng.normal(0, K ** -0.5, ((Hq + 2 * Hkv) * D, K)))
    Wgu = bf(rng.normal(0, K ** -0.5, (2 * I, K)))
    # row-parallel o_proj: this rank's K slice, its partial output rounded to bf16 (as a GPU writes it)
    ks = tp.row_split(Ko, rank, world)
    part = torch.from_numpy(bf(oracle.projection(a[:, ks], Wo[:, ks])))
    parts = [torch.empty_like(part) for _ in range(world)]
    dist.all_gather(parts, part)
    x = oracle.tp_allreduce([p.numpy() for p in parts])
    # column-parallel QKV and gate/up on this rank's rows
    rows = tp.qkv_rows(Hq, Hkv, D, rank, world)
    o = oracle.add_norm_qkv(x, resid, gamma, None, "rmsnorm", eps, Wqkv[rows], None, Hq // world, Hkv // world, D)
    grow = tp.swiglu_rows(I, rank, world)
    s = oracle.add_norm_swiglu(x, resid, gamma, None, "rmsnorm", eps, Wgu[grow], None, I // world)
    shard = torch.from_numpy(np.concatenate([o["q"].ravel(), o["k"].ravel(), o["v"].ravel(), s["out"].ravel()]))
    shards = [torch.empty_like(shard) for _ in range(world)]
    dist.all_gather(shards, shard)
    if rank == 0:
        # the single-rank computation: full o_proj partials summed the same way, all heads, all rows
        full_parts = [bf(oracle.projection(a[:, tp.row_split(Ko, r, world)], Wo[:, tp.row_split(Ko, r, world)]))
                      for r in range(world)]
        assert np.array_equal(x, oracle.tp_allreduce(full_parts))
        assert np.max(np.abs(x - bf(a @ Wo.T))) <= 2 ** -6 * np.max(np.abs(a @ Wo.T))
        ref = oracle.add_norm_qkv(x, resid, gamma, None, "rmsnorm", eps, Wqkv, None, Hq, Hkv, D)
        refs = oracle.add_norm_swiglu(x, resid, gamma, None, "rmsnorm", eps, Wgu, None, I)
        nq, nk = (Hq // world) * M * D, (Hkv // world) * M * D
        ni = M * (I // world)
        for r, sh in enumerate(shards):
            sh = sh.numpy()
            q = sh[:nq].reshape(Hq // world, M, D)
            k = sh[nq:nq + nk].reshape(Hkv // world, M, D)
            v = sh[nq + nk:nq + 2 * nk].reshape(Hkv // world, M, D)
            sw = sh[nq + 2 * nk:].reshape(M, I // world)
            hq, hk = Hq // world, Hkv // world
            assert np.allclose(q, ref["q"][r * hq:(r + 1) * hq], rtol=0, atol=1e-12)
            assert np.allclose(k, ref["k"][r * hk:(r + 1) * hk], rtol=0, atol=1e-12)
            assert np.allclose(v, ref["v"][r * hk:(r + 1) * hk], rtol=0, atol=1e-12)
            assert np.allclose(sw, refs["out"][:, r * (I // world):(r + 1) * (I // world)], rtol=0, atol=1e-12)
            assert nq + 2 * nk + ni == sh.size
        out["ok"] = True
    dist.barrier()
    dist.destroy_process_group()


def test_tensor_parallel_layout_two_gloo_ranks():
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
    assert out.get("ok")


def test_tp_layout_rejects_uneven_splits():
    sys.path.insert(0, ROOT)
    from transformer_layer_residual_b200 import tp
    import pytest
    with pytest.raises(ValueError):
        tp.qkv_rows(6, 2, 8, 0, 4)
    with pytest.raises(ValueError):
        tp.row_split(10, 2, 2)
    assert tp.swiglu_rows(4, 1, 2) == [2, 3, 6, 7]
    assert tp.qkv_rows(2, 1, 2, 0, 1) == [0, 1, 2, 3, 4, 5, 6, 7]
    assert tp.qkv_rows(4, 2, 1, 1, 2) == [2, 3, 5, 7]
