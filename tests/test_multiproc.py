"""Multi-process host logic of the benchmark, on CPU (gloo, world size 2).

The layer shards by tokens: every rank runs the whole hot path on its own batch
with replicated weights. The forward's only cross-rank step is the timing
reduction (max over ranks of the step time); the backward's is the sum of the
adapter gradients over ranks (dp.allreduce_adapter_grads, one all-reduce of a
flat buffer per layer). These tests pin both reductions, the per-rank batch
choice and the whole-job metric; the reference arm's N>1 behaviour (rank 0 alone
runs and prints) is checked on a tiny workload.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 3.0 + 2.0 * rank                       # rank 1 is the slow one
        got = bench.max_over_ranks(local_ms, torch.device("cpu"), True)
        cfg = synth.TINY
        seed = bench.rank_token_seed(cfg, rank)
        xb = synth.make_tokens(cfg.T, cfg.d, seed)
        digest = int(np.asarray(xb, dtype=np.uint64).sum())
        out[rank] = (got, seed, digest)
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction_and_batches():
    port = 29500 + (os.getpid() % 2000)
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    (m0, s0, d0), (m1, s1, d1) = out[0], out[1]
    assert m0 == m1 == 5.0                  # every rank reports the slowest rank's time
    assert s0 != s1 and d0 != d1            # independent token batches per rank
    # whole-job value: both ranks' tokens over the max-over-ranks time
    assert bench.weak_scaling_value(2, 8192, 5.0) == pytest.approx(2 * 8192 / 5e-3)


def test_single_rank_reduction_is_identity():
    assert bench.max_over_ranks(1.25, torch.device("cpu"), False) == 1.25


def _run_reference(rank, world):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                           "--steps", "1", "--warmup", "0", "--ref-sample", "2"],
                          capture_output=True, text=True, env=env, timeout=300)


def test_reference_arm_runs_on_rank0_only():
    r1 = _run_reference(1, 2)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _run_reference(0, 2)
    assert r0.returncode == 0, r0.stderr[-500:]
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
    # same metric and workload description as the GPU arm, so the two lines compare
    sys.path.insert(0, ROOT)
    import bench
    import synth
    want = bench.workload_config(synth.CONFIGS["tiny"])
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT and line["higher_is_better"] is True
    assert {k: line["config"][k] for k in want} == want


def _grad_worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    from quantized_base_lora_moe_b200.dp import FlatGrads, allreduce_adapter_grads
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        g = FlatGrads(E=4, d=64, f=128, r=8, device="cpu")
        # each rank's gradients: rank-dependent values, different per tensor
        for p in range(3):
            g.dA[p].fill_((rank + 1) * (p + 1))
            g.dB[p].fill_((rank + 1) * 10.0 * (p + 1))
        g.dA[2][1, 3, 5] = 1000.0 * (rank + 1)           # one distinct element, to catch offset mix-ups
        assert allreduce_adapter_grads(g) is None
        s = sum(i + 1 for i in range(world))
        ok = all(bool(torch.all(g.dB[p] == s * 10.0 * (p + 1))) for p in range(3))
        ok &= bool(torch.all(g.dA[0] == s)) and bool(torch.all(g.dA[1] == 2 * s))
        ok &= float(g.dA[2][1, 3, 5]) == 1000.0 * s and float(g.dA[2][1, 3, 4]) == 3 * s
        # asynchronous form: the handle completes the same sum
        g.zero_()
        g.dB[1].fill_(rank + 0.5)
        work = allreduce_adapter_grads(g, async_op=True)
        work.wait()
        ok &= bool(torch.all(g.dB[1] == sum(i + 0.5 for i in range(world)))) and float(g.flat.abs().sum()) == \
            float(g.dB[1].abs().sum())
        out[rank] = ok
    finally:
        dist.destroy_process_group()


def test_adapter_gradient_allreduce_two_ranks():
    port = 31500 + (os.getpid() % 2000)
    out = mp.Manager().dict()
    mp.spawn(_grad_worker, args=(2, port, out), nprocs=2, join=True)
    assert out[0] and out[1]


def test_flat_gradient_views_alias_one_buffer():
    from quantized_base_lora_moe_b200.dp import FlatGrads, allreduce_adapter_grads
    g = FlatGrads(E=3, d=128, f=256, r=16, device="cpu")
    n = 3 * 16 * (128 + 128 + 256) + 3 * 16 * (256 + 256 + 128)
    assert g.flat.numel() == n
    base = g.flat.data_ptr()
    for t in g.dA + g.dB:
        assert t.data_ptr() % 32 == 0 and base <= t.data_ptr() < base + 4 * n
        t.fill_(1.0)
    assert float(g.flat.sum()) == n                           # the views tile the buffer exactly
    for p in range(3):
        assert g.struct.dA[p] == g.dA[p].data_ptr() and g.struct.dB[p] == g.dB[p].data_ptr()
    assert allreduce_adapter_grads(g) is None                 # no process group: nothing to exchange
    import quantized_base_lora_moe_b200 as Q
    assert Q._grads(g) is g.struct                            # the backward calls take a FlatGrads as well
    r0 = FlatGrads(E=3, d=128, f=256, r=0, device="cpu")
    assert r0.flat.numel() == 0 and allreduce_adapter_grads(r0) is None


class _OracleAdamW:
    """CPU stand-in for AdapterAdamW in the gloo test: the oracle's AdamW on a
    master copy in the flat gradient layout."""

    def __init__(self, flat_init):
        self.p = flat_init.astype(np.float64)
        self.m = np.zeros_like(self.p)
        self.v = np.zeros_like(self.p)
        self.t = 0

    def step(self, grads):
        from oracle import tqp_oracle as O
        self.t += 1
        self.p, self.m, self.v = O.adamw_step(self.p, self.m, self.v, grads.flat.numpy().astype(np.float64), 1e-3,
                                              0.9, 0.999, 1e-8, 0.01, self.t)


def _dp_step_worker(rank, world, port, out):
    """Each rank: the oracle's layer backward on its own token shard as the local
    step, one all-reduce, the optimizer step; reports the summed gradient and
    the updated parameters."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    from oracle import tqp_oracle as O
    from quantized_base_lora_moe_b200.dp import FlatGrads, adapter_dp_step
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cfg = synth.LayerConfig("dp", T=96, d=64, E=6, k=2, f=64, g=32, r=8)
        raw = synth.make_layer(cfg)
        L = O.Layer(raw)
        x = O.bf16_to_f64(synth.make_tokens(cfg.T, cfg.d, 7))
        dy = synth.make_grad(cfg.T, cfg.d, 8, "dy1").astype(np.float64)
        shard = slice(rank * cfg.T // world, (rank + 1) * cfg.T // world)
        g = FlatGrads(cfg.E, cfg.d, cfg.f, cfg.r, device="cpu")

        def local_backward(grads):
            _, dA, dB = O.layer_backward(x[shard], dy[shard], L)
            for p in range(3):
                grads.dA[p].copy_(torch.from_numpy(dA[p]))
                grads.dB[p].copy_(torch.from_numpy(dB[p]))

        lora = np.concatenate([O.bf16_to_f64(raw[f"la{p}"]).ravel() for p in range(3)] +
                              [O.bf16_to_f64(raw[f"lb{p}"]).ravel() for p in range(3)])
        opt = _OracleAdamW(lora)
        adapter_dp_step(local_backward, g, opt)
        out[rank] = (g.flat.numpy().copy(), opt.p.copy())
    finally:
        dist.destroy_process_group()


def test_data_parallel_step_sums_shards_to_the_full_batch_gradient():
    from oracle import tqp_oracle as O
    port = 33500 + (os.getpid() % 2000)
    out = mp.Manager().dict()
    mp.spawn(_dp_step_worker, args=(2, port, out), nprocs=2, join=True)
    (g0, p0), (g1, p1) = out[0], out[1]
    assert np.array_equal(g0, g1) and np.array_equal(p0, p1)     # identical replicas after the step
    # the summed gradient is the gradient over the union of the shards
    cfg = synth.LayerConfig("dp", T=96, d=64, E=6, k=2, f=64, g=32, r=8)
    L = O.Layer(synth.make_layer(cfg))
    x = O.bf16_to_f64(synth.make_tokens(cfg.T, cfg.d, 7))
    dy = synth.make_grad(cfg.T, cfg.d, 8, "dy1").astype(np.float64)
    _, dA, dB = O.layer_backward(x, dy, L)
    full = np.concatenate([a.ravel() for a in dA] + [b.ravel() for b in dB])
    assert np.max(np.abs(g0 - full)) <= 1e-5 * np.max(np.abs(full))   # fp32 buffer of fp64 sums
