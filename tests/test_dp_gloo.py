"""World-size-2 gloo test of the data-parallel step's host logic on CPU: each
rank takes its own token shard, computes the STE weight gradients (the
oracle stands in for the GPU step here), and the all-reduce yields the
gradient of the concatenated batch; the max-over-ranks timing is the max."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle as o
        from quantization_aware_tiny_b200 import dp
        from quantization_aware_tiny_b200 import synthetic as sy
        c = sy.head_mlp_case(T=64, vocab=64, d=32, H=64, seed=dp.shard_seed(0, rank))
        shared = sy.head_mlp_case(T=1, vocab=64, d=32, H=64, seed=123)  # same weights on all ranks
        qe, qf, qp = (o.quantize_weight(shared["Wemb"], 8), o.quantize_weight(shared["Wfc"], 6),
                      o.quantize_weight(shared["Wproj"], 6))
        r = o.head_mlp_step(qe, qf, qp, c["X"].float().numpy(), c["dLogits"].float().numpy())
        grads = [torch.from_numpy(r[k].copy()) for k in ("dWemb", "dWfc", "dWproj")]
        dp.allreduce_grads(grads, dist)
        mx = dp.max_over_ranks(10.0 + rank, dist, "cpu")
        if rank == 0:
            out.put(([g.numpy() for g in grads], mx))
    finally:
        dist.destroy_process_group()


def test_dp_allreduce_equals_full_batch_gradient():
    import oracle as o
    from quantization_aware_tiny_b200 import dp
    from quantization_aware_tiny_b200 import synthetic as sy
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    grads, mx = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    shards = [sy.head_mlp_case(T=64, vocab=64, d=32, H=64, seed=dp.shard_seed(0, r)) for r in range(2)]
    shared = sy.head_mlp_case(T=1, vocab=64, d=32, H=64, seed=123)
    qe, qf, qp = (o.quantize_weight(shared["Wemb"], 8), o.quantize_weight(shared["Wfc"], 6),
                  o.quantize_weight(shared["Wproj"], 6))
    X = np.concatenate([s["X"].float().numpy() for s in shards])
    dL = np.concatenate([s["dLogits"].float().numpy() for s in shards])
    full = o.head_mlp_step(qe, qf, qp, X, dL)
    for g, k in zip(grads, ("dWemb", "dWfc", "dWproj")):
        assert np.allclose(g, full[k], rtol=1e-12, atol=1e-12), k
    assert mx == 11.0


def _sync_worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from quantization_aware_tiny_b200 import dp
        g = torch.Generator().manual_seed(100 + rank)
        head = torch.randn(64, 32, generator=g)
        fc, proj = torch.randn(16, 32, generator=g), torch.randn(32, 16, generator=g)
        mine = [head.clone(), fc.clone(), proj.clone()]
        sync = dp.GradSync(dist)
        sync.start([head])           # as soon as the head's backward is queued
        busy = torch.randn(256, 256, generator=g) @ torch.randn(256, 256, generator=g)  # "MLP backward"
        sync.start([fc, proj])       # the MLP's gradients at the end of the step
        sync.wait()
        if rank == 0:
            out.put(([t.numpy() for t in (head, fc, proj)], [t.numpy() for t in mine], float(busy.sum())))
        else:
            out.put(([t.numpy() for t in mine], None, None))
    finally:
        dist.destroy_process_group()


def test_grad_sync_overlapped_sums_equal_plain_sums():
    """GradSync (the head gradient's sum started before the MLP backward, the
    MLP's after it, one wait) gives every rank the plain sum of all ranks'
    gradients, as the serial all-reduce did."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sync_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    summed = next(g for g in got if g[1] is not None)
    other = next(g for g in got if g[1] is None)[0]
    for s, a, b in zip(summed[0], summed[1], other):
        assert np.allclose(s, a + b, rtol=0, atol=1e-5)
