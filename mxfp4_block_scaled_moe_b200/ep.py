"""Expert parallelism of the MXFP4 MoE layer over the ranks of a torch.distributed group.

The pages run GPT-OSS over several GPUs ("amd/gpt-oss-20b-MoE-Quant-W-MXFP4-A-FP8-KV-FP8",
Evaluation: tensor parallel 1-8; "gpt-oss-120b-mxfp4-fp8attn-v2", Serving: four GPUs).
For the expert layer the natural split is by expert: rank r owns experts
[r * E/G, (r + 1) * E/G) with their packed weights, and every rank routes its own tokens
with the replicated router. One step on every rank:

 1. route: top-k expert ids idx (T, k) and gates w (T, k)  (library: moe_route_topk);
 2. plan: every (token t, slot j) pair p = t*k + j goes to the owner of its expert; pairs
    are sent in order of expert id (hence of destination rank), ties in pair order;
 3. exchange the per-destination counts, then the pairs' activation rows and expert ids
    (all_to_all_single with those splits; NCCL between GPUs, gloo on CPU);
 4. the owner groups the rows it received by local expert (stable, sources in rank order)
    and runs its experts on them  (library: moe_mxfp4_experts, fp32 rows);
 5. the rows go back by the reverse exchange, in the order they were sent;
 6. each token's k expert outputs are summed with its gates in ascending expert id, fp32,
    one bf16 rounding  (library: moe_combine, given each pair's position in the send order).

Step 6 follows the single-GPU layer's order, and every expert row depends only on its own
activation row, so the result equals the single-GPU layer's bit for bit when both run the
same expert kernels. The index arithmetic here (argsort, bincount, gathers into send
buffers) is host-side plumbing on small integer tensors around the exchange; the layer's
arithmetic stays in the library's kernels, or in whatever `compute` / `combine` the caller
passes (the CPU tests pass the oracle's).
"""
from __future__ import annotations

import dataclasses

import torch
import torch.distributed as dist


def experts_per_rank(E: int, world: int) -> int:
    if E % world:
        raise ValueError(f"E = {E} experts do not split evenly over {world} ranks")
    return E // world


@dataclasses.dataclass
class DispatchPlan:
    order: torch.Tensor        # (P,) int64: the pair sent at each send position
    send_pos: torch.Tensor     # (P,) int32: the send position of each pair (t*k + j)
    send_counts: torch.Tensor  # (world,) int64: pairs per destination rank


def dispatch_plan(idx: torch.Tensor, E: int, world: int) -> DispatchPlan:
    """Send order of the (token, slot) pairs of topk ids idx (T, k): by expert id (the
    owner ranks hold contiguous expert ranges, so this also groups by destination), ties in
    pair order."""
    per = experts_per_rank(E, world)
    flat = idx.reshape(-1).to(torch.int64)
    P = flat.numel()
    pair = torch.arange(P, dtype=torch.int64, device=flat.device)
    order = torch.argsort(flat * P + pair)
    send_pos = torch.empty(P, dtype=torch.int32, device=flat.device)
    send_pos[order] = pair.to(torch.int32)
    send_counts = torch.bincount(flat // per, minlength=world)
    return DispatchPlan(order, send_pos, send_counts)


def receive_grouping(local_expert: torch.Tensor, E_local: int):
    """Rows received from every rank (source ranks in order, each ordered by expert) ->
    the stable permutation that groups them by local expert, and the expert offsets."""
    R = local_expert.numel()
    key = local_expert.to(torch.int64) * max(R, 1) + torch.arange(R, dtype=torch.int64, device=local_expert.device)
    perm = torch.argsort(key)
    counts = torch.bincount(local_expert.to(torch.int64), minlength=E_local)
    offsets = torch.zeros(E_local + 1, dtype=torch.int32, device=local_expert.device)
    offsets[1:] = torch.cumsum(counts, 0).to(torch.int32)
    return perm, offsets


def _exchange(t: torch.Tensor, send_counts, recv_counts, group):
    out = torch.empty((int(sum(recv_counts)),) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    dist.all_to_all_single(out, t.contiguous(), output_split_sizes=list(recv_counts),
                           input_split_sizes=list(send_counts), group=group)
    return out


def ep_forward(x, idx, w, E, compute, combine, group=None):
    """One expert-parallel step on this rank, given its tokens x (T, H), their routing
    idx / w (T, k) and:
      compute(rows (R, H), local expert ids (R,), offsets (E_local + 1)) -> y (R, H) fp32,
          rows grouped by local expert (offsets as moe_mxfp4_experts takes them);
      combine(y_back (P, H) fp32, idx, w, send_pos) -> out (T, H), y_back in send order.
    Every rank takes the same collective steps in the same order."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    per = experts_per_rank(E, world)
    T, k = idx.shape
    plan = dispatch_plan(idx, E, world)
    send_counts = plan.send_counts.to(torch.int64)
    recv_counts_t = torch.empty_like(send_counts)
    dist.all_to_all_single(recv_counts_t, send_counts, group=group)
    sc = send_counts.cpu().tolist()
    rc = recv_counts_t.cpu().tolist()
    token = torch.div(plan.order, k, rounding_mode="floor")
    send_rows = x[token]
    send_eid = idx.reshape(-1)[plan.order].to(torch.int32)
    recv_rows = _exchange(send_rows, sc, rc, group)
    recv_eid = _exchange(send_eid, sc, rc, group)
    local = recv_eid.to(torch.int64) - rank * per
    perm, offsets = receive_grouping(local, per)
    y_grouped = compute(recv_rows[perm].contiguous(), local[perm], offsets)
    y_recv = torch.empty_like(y_grouped)
    y_recv[perm] = y_grouped
    y_back = _exchange(y_recv, rc, sc, group)
    return combine(y_back, idx, w, plan.send_pos)


def gpu_compute(local_weights, act_scale=None, stream=None):
    """compute() for ep_forward on a GPU: the library's grouped expert GEMMs over this
    rank's experts (local_weights: gu_blocks, gu_scales, gu_bias, d_blocks, d_scales,
    d_bias of its E_local experts)."""
    from . import binding as B

    def run(rows, local_ids, offsets):
        return B.moe_mxfp4_experts(rows, offsets, *local_weights, act_scale=act_scale, stream=stream)

    return run


def gpu_combine(stream=None):
    """combine() for ep_forward on a GPU: the library's ordered weighted combine."""
    from . import binding as B

    def run(y_back, idx, w, send_pos):
        return B.moe_combine(y_back, idx, w, send_pos, stream=stream)

    return run
