"""Expert parallelism of the layer on CPU: world size 2 and 4 over gloo, each rank owning a
contiguous range of experts, against the single-rank oracle, bit for bit.

Page context: the pages run GPT-OSS over several GPUs ("amd/gpt-oss-20b-MoE-Quant-W-MXFP4-
A-FP8-KV-FP8", Evaluation, TP 1-8); the split here is by expert with an all-to-all
exchange of rows each way. The per-pair expert FFN is the oracle's, the combine an
ascending-expert fp32 sum written here; every rank routes its own tokens with the oracle.
The exchange and the index arithmetic are mxfp4_block_scaled_moe_b200.ep's.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.dirname(os.path.abspath(__file__))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _case(fp8):
    import oracle
    from helpers import pack
    from mxfp4_block_scaled_moe_b200 import inputs
    p = pack(inputs.small_layer(E=8, k=3, T=48, H=64, I=96, seed=17, router_bias=True))
    s = oracle.calibrate(p.x, p.router_w, p.router_b, *p.weights, 3) if fp8 else None
    return p, s


def _ascending_combine(y_back, idx, w, send_pos):
    y = y_back.numpy()
    idx, w, pos = idx.numpy(), w.numpy(), send_pos.numpy()
    T, k = idx.shape
    out = np.zeros((T, y.shape[1]), np.float32)
    for t in range(T):
        for j in np.argsort(idx[t], kind="stable"):
            out[t] = out[t] + np.float32(w[t, j]) * y[pos[t * k + j]]
    return torch.from_numpy(out)


def _worker(rank, world, port, fp8, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, TESTS)
    import oracle
    from mxfp4_block_scaled_moe_b200 import ep
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        p, s = _case(fp8)
        E, k = p.lay.E, p.lay.k
        per = E // world
        # this rank's tokens: a contiguous share of the batch (ranks get different counts)
        T = p.x.shape[0]
        cuts = [0] + [T * (r + 1) // world + (3 if r == 0 and world > 1 else 0) for r in range(world)]
        cuts[-1] = T
        rows = slice(cuts[rank], cuts[rank + 1])
        xb = p.x[rows]
        idx, w = oracle.topk_softmax(oracle.router_logits(xb, p.router_w, p.router_b), k)
        lo = rank * per
        wl = tuple(a[lo:lo + per] for a in p.weights)   # only this rank's experts

        def compute(rows_, local_ids, offsets):
            y = oracle.expert_rows(rows_.numpy().astype(np.uint16), local_ids.numpy().astype(np.int32), *wl,
                                   act_scale=s)
            return torch.from_numpy(y)

        x_t = torch.from_numpy(xb.astype(np.int32))   # bf16 bits, widened for gloo's all-to-all
        out = ep.ep_forward(x_t, torch.from_numpy(idx), torch.from_numpy(w), E, compute, _ascending_combine)
        q.put((rank, cuts[rank], out.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,fp8", [(2, False), (2, True), (4, False)])
def test_expert_parallel_layer_equals_the_single_rank_oracle(world, fp8):
    sys.path.insert(0, TESTS)
    p, s = _case(fp8)
    _, acc, _, _ = p.oracle_forward(act_scale=s)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, fp8, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    got = [q.get(timeout=120) for _ in range(world)]
    for pr in procs:
        pr.join(120)
        assert pr.exitcode == 0
    out = np.concatenate([g[2] for g in sorted(got)], axis=0)
    assert np.array_equal(out.view(np.uint32), acc.view(np.uint32))


def test_dispatch_plan_orders_by_expert_and_inverts():
    sys.path.insert(0, ROOT)
    from mxfp4_block_scaled_moe_b200 import ep
    idx = torch.tensor([[5, 1], [0, 7], [1, 6], [4, 5]], dtype=torch.int32)
    plan = ep.dispatch_plan(idx, E=8, world=4)
    flat = idx.reshape(-1)
    sent = flat[plan.order]
    assert sent.tolist() == sorted(flat.tolist())                  # ascending expert = destination order
    assert plan.send_counts.tolist() == [3, 0, 3, 2]               # experts {0,1},{2,3},{4,5},{6,7}
    assert torch.equal(plan.order[plan.send_pos.long()], torch.arange(8))
    # equal experts keep pair order: pairs 1 (t=0, j=1) and 4 (t=2, j=0) both go to expert 1
    pos = plan.send_pos.tolist()
    assert pos[1] < pos[4]
    perm, offsets = ep.receive_grouping(torch.tensor([1, 0, 1, 0, 0]), 2)
    assert perm.tolist() == [1, 3, 4, 0, 2] and offsets.tolist() == [0, 3, 5]
    with pytest.raises(ValueError):
        ep.dispatch_plan(idx, E=8, world=3)
