"""The data-parallel exchange on CPU: two gloo ranks, each with its own token
shard of one global batch ("Sparse-BitNet：1.58-bit 大模型天然兼容半结构化稀疏",
方法步骤详情, Algorithm 1 steps (7) and (8)).

Each rank computes the oracle's dW over its shard into the package's
GradBucket, sums it over the ranks with GradExchange (the same host code the
GPU path runs over NCCL), then applies the oracle's AdamW step with the
global clip norm.  The summed dW must equal the oracle's dW over the whole
batch (within the rounding of one fp32 add), and both replicas must end with
bit-identical W, m, v, W_eff, gamma, masks and flip counts."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synth
from semi_structured_sparsity_step_b200.data_parallel import GradBucket, GradExchange

SHAPES = {"qkv": (64, 128), "down": (48, 64)}
T_GLOBAL = 96
N, M = 6, 8


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _global_batch():
    """The whole batch, identical on every rank (seeded)."""
    W, X, dY = {}, {}, {}
    for i, (name, (d_out, d_in)) in enumerate(SHAPES.items()):
        W[name] = synth.bits(synth.trimodal_weight(d_out, d_in, seed=40, tensor_id=i))
        X[name] = synth.bits(synth.activations(T_GLOBAL, d_in, seed=40, tensor_id=100 + i))
        dY[name] = synth.bits(synth.grad_output(T_GLOBAL, d_out, seed=40, tensor_id=200 + i))
    return W, X, dY


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        W, X, dY = _global_batch()
        share = T_GLOBAL // world
        sl = slice(rank * share, (rank + 1) * share)
        bucket = GradBucket(SHAPES, "cpu")
        ex = GradExchange(bucket)
        assert ex.active
        for name in SHAPES:                       # backward of this rank's shard, exchange per projection
            bucket[name].copy_(torch.from_numpy(oracle.backward_dw(dY[name][sl], X[name][sl])))
            ex.launch(name)
        ex.wait()
        reduced = {name: bucket[name].numpy().copy() for name in SHAPES}
        S = oracle.grad_sqnorm(*reduced.values())
        clip = oracle.grad_clip_scale(S, 1.0)
        sc = oracle.adamw_scalars(1e-3, 0.9, 0.95, 1e-5, 0.1, step=3)
        res = {}
        for name, (d_out, d_in) in SHAPES.items():
            m = np.full((d_out, d_in), 1e-4, np.float32)
            v = np.full((d_out, d_in), 1e-6, np.float32)
            r = oracle.adamw_weight_step(W[name], reduced[name], m, v, N, M, sc, clip)
            res[name] = {k: (np.asarray(val).tobytes() if not isinstance(val, (int, float)) else val)
                         for k, val in r.items() if val is not None}
        out[rank] = {"reduced": {k: v.tobytes() for k, v in reduced.items()}, "step": res,
                     "clip": float(clip), "S": S}
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_two_ranks_sum_dw_and_apply_identical_updates():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    r0, r1 = out[0], out[1]
    # every replica holds the same summed gradient and the same new state, bit for bit
    assert r0["reduced"] == r1["reduced"]
    assert r0["step"] == r1["step"]
    assert r0["clip"] == r1["clip"] and r0["S"] == r1["S"]
    # the sum over ranks is dW of the concatenated batch
    W, X, dY = _global_batch()
    u = 2.0 ** -24
    for name, (d_out, d_in) in SHAPES.items():
        got = np.frombuffer(r0["reduced"][name], np.float32).reshape(d_out, d_in).astype(np.float64)
        ref = oracle.backward_dw(dY[name], X[name]).astype(np.float64)
        absb = np.abs(oracle.bf16_to_f32(dY[name]).astype(np.float64)).T @ \
            np.abs(oracle.bf16_to_f32(X[name]).astype(np.float64))
        assert (np.abs(got - ref) <= 4 * u * absb + u * np.abs(ref)).all(), name
    # and the update moved the weights (the exchange fed a real step)
    st = r0["step"]["qkv"]
    assert st["w_bits"] != W["qkv"].tobytes()


def test_single_process_exchange_is_a_no_op():
    bucket = GradBucket(SHAPES, "cpu")
    bucket["qkv"].fill_(1.5)
    ex = GradExchange(bucket)
    assert not ex.active
    ex.launch_all()
    ex.wait()
    assert torch.all(bucket["qkv"] == 1.5)
    assert torch.all(bucket["down"] == 0.0)


def test_bucket_views_are_disjoint_aligned_and_cover_every_projection():
    shapes = {"q": (2048, 2048), "k": (256, 2048), "gate": (11008, 2048), "down": (2048, 11008), "odd": (8, 16)}
    b = GradBucket(shapes, "meta")
    seen = 0
    for name, (d_out, d_in) in shapes.items():
        o, n = b.offsets[name]
        assert n == d_out * d_in and (o * 4) % 16 == 0
        assert b[name].shape == (d_out, d_in)
        assert o >= seen
        seen = o + n
    assert seen <= b.numel
