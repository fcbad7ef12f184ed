"""Context sharding of one LCA decode step across ranks.

Each rank holds a slice of every sequence's cache -- tokens [pos0, pos0 +
n_tok) of a context of L tokens, cut on group boundaries inside the condensed
part -- and computes the partial softmax sums (M, Z, O) of the entries it
holds (lca_decode_partial).  The partials of all ranks are exchanged (an
all-gather of B*H*(d_c+2) floats per rank: NCCL on GPUs, gloo on CPU) and
merged exactly by the online-softmax merge (lca_merge_partials): the method
of the Pulsar Attention page, "Fase 2" (per-host attention, then a merge of
the per-host softmax statistics).  Every rank ends with the whole output.
"""
from __future__ import annotations


def slice_bounds(L: int, g: int, w: int, parts: int) -> list[tuple[int, int]]:
    """Cut tokens [0, L) into `parts` contiguous slices of about equal length
    whose bounds inside the condensed part [0, n_G g) are multiples of g (no
    group is cut).  Returns [(pos0, n_tok)]; a slice may be empty."""
    nG = (L - w) // g if L > w else 0
    win0 = nG * g
    bounds = [0]
    for i in range(1, parts):
        t = (L * i) // parts
        if t < win0:
            t = (t // g) * g
        bounds.append(max(t, bounds[-1]))
    bounds.append(L)
    return [(bounds[i], bounds[i + 1] - bounds[i]) for i in range(parts)]


def exchange_partials(part_mz, part_o, group=None):
    """All-gather this rank's partials ([B,H,2] and [B,H,d_c] tensors, on the
    device the backend serves) and return them stacked over ranks
    ([world,B,H,2], [world,B,H,d_c]).  Without a process group: this rank's
    alone."""
    import torch
    import torch.distributed as dist
    if group is None and not (dist.is_available() and dist.is_initialized()):
        return part_mz[None], part_o[None]
    world = dist.get_world_size(group)
    mz = [torch.empty_like(part_mz) for _ in range(world)]
    o = [torch.empty_like(part_o) for _ in range(world)]
    dist.all_gather(mz, part_mz.contiguous(), group=group)
    dist.all_gather(o, part_o.contiguous(), group=group)
    return torch.stack(mz), torch.stack(o)


def context_sharded_decode(plan, q_c, q_r, c_slice, k_slice, pos0: int, L: int, g: int, w: int,
                           group=None, stream=None):
    """One rank's share of a context-sharded LCA decode on its GPU: the partial
    over its slice (c_slice [B,n_tok,d_c], k_slice [B,n_tok,d_r] = tokens
    [pos0, pos0 + n_tok) of each sequence), the exchange, the merge.  Returns
    (out [B,H,d_c] float32, the slice's anchors [B,H,n_slice_groups] int32)."""
    import torch
    from . import slice_groups
    B, H, d_c = q_c.shape
    n_tok = c_slice.shape[1]
    ng = slice_groups(L, g, w, pos0, n_tok)
    mz = torch.empty(B, H, 2, dtype=torch.float32, device=q_c.device)
    po = torch.empty(B, H, d_c, dtype=torch.float32, device=q_c.device)
    anc = torch.empty(B, H, max(ng, 1), dtype=torch.int32, device=q_c.device)
    plan.decode_partial(q_c, q_r, c_slice, k_slice, n_tok, pos0, L, g, w, mz, po,
                        anc if ng > 0 else None, stream)
    all_mz, all_o = exchange_partials(mz, po, group)
    out = torch.empty(B, H, d_c, dtype=torch.float32, device=q_c.device)
    plan.merge_partials(all_mz.shape[0], all_mz, all_o, out, stream)
    return out, anc[:, :, :ng]
