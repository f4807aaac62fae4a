"""Expert-parallel, tensor-parallel and all-to-all forward of one MoE layer.

Every arithmetic step runs in libmoe_b200.so's kernels.  Between ranks this
module uses torch.distributed (NCCL on GPUs): one all-reduce of an fp32
partial output (expert and tensor parallelism), or uneven all-to-all
exchanges of token rows (the all-to-all dispatcher).

* Expert parallelism, masked-local plus all-reduce (metrale ep_dispatch.rs,
  module doc: "The served EP MoE is masked-local plus all-reduce"; diffulex.moe
  API reference, ``EPFusedMoE``).  Rank r of R owns the contiguous experts
  ``expert_range(E, R, r)``; it routes and dispatches its whole batch, gathers
  and runs only its experts' rows, merges them into an fp32 partial (the
  other ranks' experts contribute nothing there), the partials are summed
  across ranks and rounded once.
* Tensor parallelism (diffulex.moe API reference, ``TPFusedMoE``; the
  modelexpress refit test's ``INTER_PER_TP`` slices: rank r takes rows
  ``[r*I/tp, (r+1)*I/tp)`` of each of w1 and w3, "w1 low, w3 high" in its
  ``[E, 2*I/tp, H]`` slot).  w2 is split along its I columns the same way.
  Every rank runs every expert on its I-slice; the partial outputs add up.
* All-to-all dispatcher (diffulex.moe API reference, ``NaiveA2ADispatcher``:
  a dispatcher that moves tokens between ranks for expert execution).  Each
  rank sends every assignment's token row to the rank that owns its expert,
  the owner runs its experts on what it received, and the outputs travel
  back to be merged in the sender's token order.

The host-side helpers here (ranges, weight slicing, the collectives) work on
CPU tensors too, which is how their multi-rank logic is tested without GPUs.
"""
from __future__ import annotations

import torch

from . import (MoELayerBuffers, moe_combine, moe_combine_range, moe_dispatch, moe_ep_owner,
               moe_ep_pack_ids, moe_experts, moe_experts_shared, moe_finalize, moe_gather,
               moe_route)

__all__ = ["expert_range", "ep_local_params", "tp_shard_params", "allreduce_sum_",
           "all_to_all_rows", "ShardedBuffers", "moe_layer_partial_ep", "moe_layer_forward_ep",
           "moe_layer_partial_tp", "moe_layer_forward_tp", "A2ABuffers", "a2a_send",
           "a2a_experts", "a2a_merge", "moe_layer_forward_a2a", "exchange_counts"]


# ------------------------------------------------------------ host-side ---

def expert_range(E: int, world: int, rank: int):
    """Experts [start, end) of ``rank`` out of ``world``: contiguous ranges
    [floor(E*r/R), floor(E*(r+1)/R)), as the ep_dispatch.rs table's
    local_expert_start..local_expert_end (every expert on exactly one rank)."""
    if not (1 <= world <= E and 0 <= rank < world):
        raise ValueError(f"need 1 <= world <= E and 0 <= rank < world (E={E}, world={world}, "
                         f"rank={rank})")
    return E * rank // world, E * (rank + 1) // world


def ep_local_params(params: dict, start: int, end: int, run_shared: bool) -> dict:
    """What an expert-parallel rank holds: the router (replicated), experts
    [start, end) of w13 / w2, and the shared expert on the one rank that runs
    it (``run_shared``)."""
    out = {"W_gate": params["W_gate"], "bias": params.get("bias"),
           "w13": params["w13"][start:end].contiguous(),
           "w2": params["w2"][start:end].contiguous()}
    if run_shared and params.get("w13s") is not None:
        out.update(w13s=params["w13s"], w2s=params["w2s"], w_sg=params["w_sg"])
    return out


def _tp_w13(w13: torch.Tensor, rank: int, tp: int) -> torch.Tensor:
    """[..., 2I, H] fused gate/up -> [..., 2I/tp, H]: rank's rows of the gate
    half, then the same rows of the up half."""
    I = w13.shape[-2] // 2
    if I % tp:
        raise ValueError(f"I = {I} is not divisible by tp = {tp}")
    it = I // tp
    gate = w13.narrow(-2, rank * it, it)
    up = w13.narrow(-2, I + rank * it, it)
    return torch.cat([gate, up], dim=-2).contiguous()


def _tp_w2(w2: torch.Tensor, rank: int, tp: int) -> torch.Tensor:
    """[..., H, I] -> [..., H, I/tp]: the rank's columns of the down projection."""
    I = w2.shape[-1]
    it = I // tp
    return w2.narrow(-1, rank * it, it).contiguous()


def tp_shard_params(params: dict, rank: int, tp: int) -> dict:
    """What a tensor-parallel rank holds: the router and the shared expert's
    gate vector (replicated), and its I-slices of every expert (and of the
    shared expert)."""
    out = {"W_gate": params["W_gate"], "bias": params.get("bias"),
           "w13": _tp_w13(params["w13"], rank, tp), "w2": _tp_w2(params["w2"], rank, tp)}
    if params.get("w13s") is not None:
        out.update(w13s=_tp_w13(params["w13s"], rank, tp), w2s=_tp_w2(params["w2s"], rank, tp),
                   w_sg=params["w_sg"])
    return out


def _group_size(group) -> int:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return 1
    return dist.get_world_size(group)


def allreduce_sum_(t: torch.Tensor, group=None) -> torch.Tensor:
    """In-place sum of ``t`` over the ranks of ``group`` (nothing to do alone)."""
    import torch.distributed as dist
    if _group_size(group) > 1:
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return t


def all_to_all_rows(send: torch.Tensor, send_counts, recv_counts, group=None) -> torch.Tensor:
    """Rows [sum(send_counts[:q]), +send_counts[q]) of ``send`` go to rank q;
    the result holds, in rank order, the rows every rank sent here."""
    import torch.distributed as dist
    recv = send.new_empty((int(sum(recv_counts)),) + tuple(send.shape[1:]))
    if _group_size(group) == 1:
        recv.copy_(send)
        return recv
    dist.all_to_all_single(recv, send, [int(c) for c in recv_counts],
                           [int(c) for c in send_counts], group=group)
    return recv


def exchange_counts(send_counts: torch.Tensor, group=None) -> torch.Tensor:
    """Every rank's count for this rank, in rank order (all-to-all of one int each)."""
    import torch.distributed as dist
    if _group_size(group) == 1:
        return send_counts.clone()
    recv = torch.empty_like(send_counts)
    dist.all_to_all_single(recv, send_counts, group=group)
    return recv


# ------------------------------------------------------------ GPU path ---

class ShardedBuffers(MoELayerBuffers):
    """MoELayerBuffers plus the fp32 partial output the ranks add up."""

    def __init__(self, T, H, E, k, I, dtype, device="cuda", shared_I=None):
        super().__init__(T, H, E, k, I, dtype, device=device, shared_I=shared_I)
        self.partial = torch.empty(T, H, dtype=torch.float32, device=torch.device(device))


def _route_and_dispatch(x, params, k, renormalize, buf, stream, gather: bool):
    E = params["W_gate"].shape[0]
    moe_route(x, params["W_gate"], params.get("bias"), k, renormalize, buf.logits, buf.ids,
              buf.w, status=buf.status, stream=stream)
    moe_dispatch(buf.ids, buf.w, x if gather else None, E, buf.counts, buf.offsets, buf.perm,
                 buf.inv_perm, buf.packed_tok, buf.packed_w, buf.x_packed, buf.ws, buf.status,
                 stream=stream)


def moe_layer_partial_ep(x, params_local: dict, start: int, end: int, k: int,
                         renormalize: bool, buf: ShardedBuffers, stream=None):
    """This rank's fp32 partial of the expert-parallel layer, into ``buf.partial``
    (before the all-reduce).  ``params_local`` from ep_local_params."""
    _route_and_dispatch(x, params_local, k, renormalize, buf, stream, gather=False)
    moe_gather(x, buf.packed_tok, buf.offsets, start, end, buf.x_packed, status=buf.status,
               stream=stream)
    offs = buf.offsets[start:]                   # absolute rows: a valid table for [start, end)
    shared = sg = None
    if params_local.get("w13s") is not None:
        moe_route(x, params_local["w_sg"].view(1, -1), None, 0, False, buf.sg_logit,
                  status=buf.status, stream=stream)
        moe_experts_shared(buf.x_packed, offs, buf.packed_w, params_local["w13"],
                           params_local["w2"], buf.h, buf.y_packed, x, params_local["w13s"],
                           params_local["w2s"], buf.sh_h, buf.sh_y, ws=buf.ws_experts,
                           status=buf.status, stream=stream)
        shared, sg = buf.sh_y, buf.sg_logit
    else:
        moe_experts(buf.x_packed, offs, buf.packed_w, params_local["w13"], params_local["w2"],
                    buf.h, buf.y_packed, ws=buf.ws_experts, status=buf.status, stream=stream)
    moe_combine_range(buf.y_packed, buf.inv_perm, buf.offsets, start, end, buf.T, k,
                      buf.partial, shared, sg, status=buf.status, stream=stream)
    return buf.partial


def moe_layer_forward_ep(x, params_local: dict, start: int, end: int, k: int,
                         renormalize: bool, buf: ShardedBuffers, group=None, stream=None):
    """Masked-local expert-parallel layer: partial, all-reduce, one rounding
    into ``buf.out``."""
    moe_layer_partial_ep(x, params_local, start, end, k, renormalize, buf, stream=stream)
    allreduce_sum_(buf.partial, group)
    moe_finalize(buf.partial, buf.out, stream=stream)
    return buf.out


def moe_layer_partial_tp(x, params_tp: dict, k: int, renormalize: bool, buf: ShardedBuffers,
                         stream=None):
    """This rank's fp32 partial of the tensor-parallel layer (``params_tp`` from
    tp_shard_params; ``buf`` sized with I/tp and I_s/tp)."""
    E = params_tp["W_gate"].shape[0]
    _route_and_dispatch(x, params_tp, k, renormalize, buf, stream, gather=True)
    shared = sg = None
    if params_tp.get("w13s") is not None:
        moe_route(x, params_tp["w_sg"].view(1, -1), None, 0, False, buf.sg_logit,
                  status=buf.status, stream=stream)
        moe_experts_shared(buf.x_packed, buf.offsets, buf.packed_w, params_tp["w13"],
                           params_tp["w2"], buf.h, buf.y_packed, x, params_tp["w13s"],
                           params_tp["w2s"], buf.sh_h, buf.sh_y, ws=buf.ws_experts,
                           status=buf.status, stream=stream)
        # the gate scales each rank's slice of the shared output; the slices add up
        shared, sg = buf.sh_y, buf.sg_logit
    else:
        moe_experts(buf.x_packed, buf.offsets, buf.packed_w, params_tp["w13"], params_tp["w2"],
                    buf.h, buf.y_packed, ws=buf.ws_experts, status=buf.status, stream=stream)
    moe_combine_range(buf.y_packed, buf.inv_perm, buf.offsets, 0, E, buf.T, k, buf.partial,
                      shared, sg, status=buf.status, stream=stream)
    return buf.partial


def moe_layer_forward_tp(x, params_tp: dict, k: int, renormalize: bool, buf: ShardedBuffers,
                         group=None, stream=None):
    """Tensor-parallel layer: partial, all-reduce, one rounding into ``buf.out``."""
    moe_layer_partial_tp(x, params_tp, k, renormalize, buf, stream=stream)
    allreduce_sum_(buf.partial, group)
    moe_finalize(buf.partial, buf.out, stream=stream)
    return buf.out


class A2ABuffers:
    """The sender-side buffers of the all-to-all layer (per-rank token batch
    T, top-k k, R ranks); receiver-side buffers grow on demand."""

    def __init__(self, T, H, E, k, world, dtype, device="cuda", shared_I=None):
        dev = torch.device(device)
        self.T, self.H, self.E, self.k, self.world = T, H, E, k, world
        self.dtype, self.device, self.shared_I = dtype, dev, shared_I
        # routing and the by-owner dispatch of this rank's assignments; the
        # merge takes the returned rows as fp32, so the shared expert's output
        # (merged beside them) is fp32 too
        self.route = MoELayerBuffers(T, H, E, k, 8, dtype, device=dev, shared_I=shared_I,
                                     y_f32=True)
        self.owner = torch.empty(T, k, dtype=torch.int32, device=dev)
        self.send = MoELayerBuffers(T, H, world, k, 8, dtype, device=dev)
        self.send_eid = torch.empty(T * k, dtype=torch.int32, device=dev)
        self.out = torch.empty(T, H, dtype=dtype, device=dev)
        self.recv = None          # MoELayerBuffers of the received rows (k = 1)
        self.recv_cap = 0


def a2a_send(x, params_local: dict, k: int, renormalize: bool, buf: A2ABuffers, stream=None):
    """Sender side: route this rank's tokens, find every assignment's owning
    rank, and dispatch by owner -- rows grouped by destination rank, in
    assignment order inside a group.  Returns (send counts [world] int32 on
    the device, token rows [T*k,H], rank-local expert ids [T*k], weights
    [T*k]); rows [offsets[q], offsets[q+1]) go to rank q."""
    E, world = buf.E, buf.world
    rb, sb = buf.route, buf.send
    moe_route(x, params_local["W_gate"], params_local.get("bias"), k, renormalize, rb.logits,
              rb.ids, rb.w, status=rb.status, stream=stream)
    moe_ep_owner(rb.ids, E, world, buf.owner, status=rb.status, stream=stream)
    moe_dispatch(buf.owner, rb.w, x, world, sb.counts, sb.offsets, sb.perm, sb.inv_perm,
                 sb.packed_tok, sb.packed_w, sb.x_packed, sb.ws, rb.status, stream=stream)
    moe_ep_pack_ids(rb.ids, sb.perm, sb.offsets, E, world, buf.send_eid, stream=stream)
    return sb.counts, sb.x_packed, buf.send_eid, sb.packed_w


def a2a_experts(x_recv, eid_recv, w_recv, params_local: dict, buf: A2ABuffers, stream=None):
    """Owner side: the rows this rank received (token rows, its own expert
    ids, routing weights) dispatched by local expert, run through its experts
    (weights applied there) and put back in the order they arrived.  Returns
    y [n_recv, H] fp32 (the executor's values exactly: k = 1 adds nothing)."""
    n_recv = x_recv.shape[0]
    y_recv = torch.empty(n_recv, buf.H, dtype=torch.float32, device=buf.device)
    if n_recv == 0:
        return y_recv
    e_loc = params_local["w13"].shape[0]
    if buf.recv is None or buf.recv_cap < n_recv:
        buf.recv = MoELayerBuffers(n_recv, buf.H, e_loc, 1, params_local["w13"].shape[1] // 2,
                                   buf.dtype, device=buf.device)
        buf.recv_cap = n_recv
    r, st = buf.recv, buf.route.status
    moe_dispatch(eid_recv.view(n_recv, 1), w_recv.view(n_recv, 1), x_recv, e_loc, r.counts,
                 r.offsets, r.perm, r.inv_perm, r.packed_tok, r.packed_w, r.x_packed, r.ws, st,
                 stream=stream)
    moe_experts(r.x_packed[:n_recv], r.offsets, r.packed_w, params_local["w13"],
                params_local["w2"], r.h[:n_recv], r.y_packed[:n_recv], ws=r.ws_experts,
                status=st, stream=stream)
    moe_combine(r.y_packed, r.inv_perm, n_recv, 1, y_recv, status=st, stream=stream)
    return y_recv


def a2a_merge(x, y_back, params_local: dict, k: int, buf: A2ABuffers, stream=None):
    """Sender side again: y_back holds, in send order, the weighted expert
    output of every assignment; merge each token's k of them in order (plus
    the shared expert, which every rank holds, on its own tokens) and round
    once into ``buf.out``."""
    rb, sb = buf.route, buf.send
    shared = sg = None
    if params_local.get("w13s") is not None:
        moe_route(x, params_local["w_sg"].view(1, -1), None, 0, False, rb.sg_logit,
                  status=rb.status, stream=stream)
        moe_experts(x, rb.sh_offsets, None, params_local["w13s"].unsqueeze(0),
                    params_local["w2s"].unsqueeze(0), rb.sh_h, rb.sh_y, ws=rb.ws_experts,
                    status=rb.status, stream=stream)
        shared, sg = rb.sh_y, rb.sg_logit
    moe_combine(y_back, sb.inv_perm, buf.T, k, buf.out, shared, sg, status=rb.status,
                stream=stream)
    return buf.out


def moe_layer_forward_a2a(x, params_local: dict, k: int, renormalize: bool, buf: A2ABuffers,
                          group=None, stream=None):
    """All-to-all expert-parallel layer on this rank's tokens x [T,H]:
    a2a_send, exchange counts and rows, a2a_experts, send the outputs back,
    a2a_merge.  The exchanges read the split sizes on the host (one
    synchronisation each way).  ``params_local`` holds the router, this
    rank's experts (ep_local_params) and the shared expert if any."""
    counts, x_send, eid_send, w_send = a2a_send(x, params_local, k, renormalize, buf,
                                                stream=stream)
    send_counts = counts.to(torch.int64)
    recv_counts = exchange_counts(send_counts, group)
    sc = send_counts.cpu().tolist()
    rc = recv_counts.cpu().tolist()
    x_recv = all_to_all_rows(x_send[:sum(sc)], sc, rc, group)
    eid_recv = all_to_all_rows(eid_send[:sum(sc)], sc, rc, group)
    w_recv = all_to_all_rows(w_send[:sum(sc)], sc, rc, group)
    y_recv = a2a_experts(x_recv, eid_recv, w_recv, params_local, buf, stream=stream)
    y_back = all_to_all_rows(y_recv, rc, sc, group)
    return a2a_merge(x, y_back, params_local, k, buf, stream=stream)
