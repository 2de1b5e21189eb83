"""Expert-parallel MoE layer forward: the kept slots travel to their experts.

The layer's experts are split over the ranks of a process group: rank r owns
experts r*E/W .. (r+1)*E/W - 1.  Each rank holds its own tokens.

1. A rank routes its tokens (``ace_moe_route``).
2. It sends every kept slot to the rank that owns the slot's expert: the
   token's expert input row, the slot's gate and the expert's local index.
3. Each rank runs its own experts on the slots it received
   (``ace_moe_experts``).
4. Each output goes back to the slot's origin rank.
5. The origin adds its tokens' slot outputs in rank order
   (``ace_moe_combine``, the combine of ``ace_moe_forward``).

Skipped slots never leave their rank, so skipping shrinks both exchanges by
the skip rate ([ACE] "Conclusion", future directions: distributed expert
dispatch).

Each way is one all-to-all of variable sizes (the counts go first), NCCL
between GPUs.  The CPU tests run the same exchange code over gloo, with the
oracle standing in for the experts and the combine.  The arithmetic is in the
injected experts and combine functions (the library's kernels on the GPU);
this module moves rows and keeps the bookkeeping of where each slot went.
"""
import torch
import torch.distributed as dist


def dispatch_plan(idx, keep, E, world):
    """This rank's kept slots in send order: (destination rank, expert, slot
    id t * k + i).  Returns the slot ids, their experts and the count per
    destination rank."""
    T, k = idx.shape
    slot = torch.nonzero(keep.reshape(-1) != 0).reshape(-1)  # (token, rank) order
    e = idx.reshape(-1)[slot].long()
    dest = e // (E // world)
    order = torch.argsort((dest * E + e) * (T * k) + slot)  # distinct keys: a total order
    slot, e, dest = slot[order], e[order], dest[order]
    return slot, e, torch.bincount(dest, minlength=world)


def ep_moe_forward(x, idx, gate, keep, E, experts_fn, combine_fn, group=None):
    """The combined expert outputs of this rank's tokens.

    x [T][d] are the experts' input rows of the rank's tokens.  idx, gate and
    keep [T][k] are their routing and mask.  experts_fn(xp, offsets, g) runs
    this rank's experts on slots grouped by local expert and returns
    g * f(xp) as [S][d]:
      - xp is [S][d];
      - offsets is [E/W + 1] int32;
      - g is [S].

    combine_fn(slot_of, rows) returns y [T][d].  rows are the outputs of this
    rank's kept slots, back from their owners.  slot_of [T][k] int32 gives
    each slot's row in rows, -1 for a skipped slot.  y adds each token's rows
    in rank order.
    """
    world = dist.get_world_size(group)
    if E % world:
        raise ValueError("%d experts do not split evenly over %d ranks" % (E, world))
    per = E // world
    T, k = idx.shape
    dev = x.device
    slot, e, send_counts = dispatch_plan(idx, keep, E, world)
    # the counts first: every rank learns how many slots it receives from each
    recv_counts = torch.empty_like(send_counts)
    dist.all_to_all_single(recv_counts, send_counts, group=group)
    sc, rc = send_counts.tolist(), recv_counts.tolist()
    n_recv = sum(rc)
    # the slots: expert input rows, the expert's index at its owner, gates
    recv_x = x.new_empty((n_recv, x.shape[1]))
    dist.all_to_all_single(recv_x, x[slot // k].contiguous(), rc, sc, group=group)
    recv_e = torch.empty(n_recv, dtype=torch.int32, device=dev)
    dist.all_to_all_single(recv_e, (e % per).to(torch.int32), rc, sc, group=group)
    recv_g = gate.new_empty(n_recv)
    dist.all_to_all_single(recv_g, gate.reshape(-1)[slot].contiguous(), rc, sc, group=group)
    # own experts on the received slots, grouped by local expert (the key
    # keeps the arrival order within an expert)
    grp = torch.argsort(recv_e.long() * max(n_recv, 1) + torch.arange(n_recv, device=dev))
    offsets = torch.zeros(per + 1, dtype=torch.int32, device=dev)
    offsets[1:] = torch.cumsum(torch.bincount(recv_e.long(), minlength=per), 0)
    yp = experts_fn(recv_x[grp].contiguous(), offsets, recv_g[grp].contiguous())
    back = torch.empty_like(yp)
    back[grp] = yp
    # the outputs home, in the order their slots left
    ret = yp.new_empty((slot.numel(), yp.shape[1]))
    dist.all_to_all_single(ret, back, sc, rc, group=group)
    slot_of = torch.full((T * k,), -1, dtype=torch.int32, device=dev)
    slot_of[slot] = torch.arange(slot.numel(), dtype=torch.int32, device=dev)
    return combine_fn(slot_of.view(T, k), ret)


def ace_experts_fn(expert_layer, ws, stream=None):
    """experts_fn over the library's expert kernels: expert_layer holds this
    rank's experts (``ace.make_expert_layer``); ws is a workspace of
    ``ace.ace_experts_workspace_size(expert_layer, max_slots)`` bytes."""
    from . import ace

    def fn(xp, offsets, g):
        yslot = torch.empty((xp.shape[0], expert_layer.d), dtype=xp.dtype, device=xp.device)
        if xp.shape[0] > 0:
            ace.ace_moe_experts(expert_layer, xp, offsets, g.float().contiguous(), yslot, ws,
                                stream=stream)
        return yslot

    return fn


def ace_combine_fn(y, ws, stream=None):
    """combine_fn over the library's combine kernel, writing y [T][d]."""
    from . import ace

    def fn(slot_of, rows):
        return ace.ace_moe_combine(slot_of.contiguous(), rows.contiguous(), y, ws, stream=stream)

    return fn


def ep_layer_forward(layer, expert_layer, u, tau, ws_route, ws_experts, group=None,
                     renorm=True, fusion="max"):
    """One layer on this rank's tokens u [T][d] with experts spread over the
    group.  ``layer`` carries the full router, gamma and tables: every rank
    routes over all E experts.  ``expert_layer`` carries this rank's E/W
    experts.  ws_route (ace_workspace_size(layer, T)) also serves the combine.
    Returns y [T][d] in u's dtype."""
    from . import ace

    T = u.shape[0]
    k = layer.k
    x = torch.empty_like(u)
    idx = torch.empty((T, k), dtype=torch.int32, device=u.device)
    gate = torch.empty((T, k), dtype=torch.float32, device=u.device)
    keep = torch.empty((T, k), dtype=torch.uint8, device=u.device)
    if T > 0:
        ace.ace_moe_route(layer, u, tau, x, idx, gate, keep, ws_route, renorm=renorm,
                          fusion=fusion)
    y = torch.empty_like(u)
    return ep_moe_forward(x, idx, gate, keep, layer.E, ace_experts_fn(expert_layer, ws_experts),
                          ace_combine_fn(y, ws_route), group=group)
