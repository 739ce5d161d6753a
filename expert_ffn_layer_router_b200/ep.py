"""Expert parallelism: the layer's E experts split over the ranks of a process group.

In "Expert Networks > Worked Example: Expert Specialization" the four experts run concurrently,
each on its own piece of hardware; the fused-MoE dataflow diagram sends each token's rows to its
experts and sums the k outputs back in token order.  Here every rank holds T_local tokens and
E / world experts (rank r owns experts [r E_l, (r + 1) E_l)), and one forward gives, for the
union of all ranks' tokens in rank order, exactly what the single-device layer gives for that
batch:

1. each rank computes its tokens' logits and top-k (no capacity yet);
2. every (token, expert) pair goes to the expert's owner as a candidate: (expert, weight);
3. the owner applies the capacity K = min(T_g, floor(C T_g k / E)) of the whole batch
   (T_g = world * T_local) to each of its experts: the candidates arrive grouped by source rank
   and, within a rank, in token order, so their order is the global token order and the
   priority (weight descending, token ascending) and slots (rank in token order) are the
   single-device ones (moe_capacity_dispatch);
4. the slots go back to the sources, which send the x rows of their kept pairs;
5. the owner runs the expert FFN on the rows it received (moe_expert_ffn);
6. the expert rows go back and each source combines its tokens (moe_combine).

Transfers are torch.distributed all-to-alls (NCCL over NVLink on GPUs, gloo on CPU).  Their
split sizes must be known on the host, so the forward synchronises the host twice: once for the
candidate counts per owner and once for the kept-row counts; all later sizes follow from those.
With one rank every exchange is the identity and copies nothing.  Every compute
step runs in the library's kernels; the plumbing between them (grouping pairs by destination,
index bookkeeping) uses torch tensor operations.  The compute steps are methods of one object
(`CudaSteps` here), so the exchange logic can be checked on CPU ranks against the oracle with the
same steps computed there.
"""
import math

import torch
import torch.distributed as dist

from . import moe


def _a2a(send, send_counts, recv_counts, group):
    """all_to_all_single along dim 0 with the given per-rank row counts (python lists).  With one
    rank the exchange is the identity and nothing is copied."""
    if dist.get_world_size(group) == 1:
        return send
    out = send.new_empty((sum(recv_counts),) + tuple(send.shape[1:]))
    dist.all_to_all_single(out, send.contiguous(), recv_counts, send_counts, group=group)
    return out


def _a2a_counts(send_counts, group):
    if dist.get_world_size(group) == 1:
        return send_counts
    recv = torch.empty_like(send_counts)
    dist.all_to_all_single(recv, send_counts.contiguous(), group=group)
    return recv


def _group_order(dest, world):
    """Positions 0..P-1 grouped by destination rank, ascending within each group (a stable
    counting sort), and the group sizes."""
    P = dest.numel()
    if P == 0:
        return dest.clone(), torch.zeros(world, dtype=torch.int64, device=dest.device)
    if world > 16:
        # The one-hot prefix sums below take P * world words; with many ranks a stable sort is
        # the smaller way to the same order.
        counts = torch.zeros(world, dtype=torch.int64, device=dest.device).scatter_add_(
            0, dest, torch.ones_like(dest))
        return torch.argsort(dest, stable=True), counts
    csum = torch.cumsum(torch.nn.functional.one_hot(dest, world), dim=0)   # [P, world]
    counts = csum[-1]
    rank_in = csum.gather(1, dest.view(-1, 1)).view(-1) - 1
    pos = (torch.cumsum(counts, 0) - counts)[dest] + rank_in
    order = torch.empty_like(dest)
    order[pos] = torch.arange(P, dtype=dest.dtype, device=dest.device)
    return order, counts


class CudaSteps:
    """The layer's steps on this rank's GPU, through the C ABI.  Workspaces are allocated once,
    for the largest problem an owner can receive."""

    def __init__(self, T_local, d_model, d_ff, E, E_local, k, K, world, dtype, device, flags):
        self.E_local, self.k, self.dtype, self.flags = E_local, k, dtype, flags
        self.d_model, self.d_ff = d_model, d_ff
        self.device = torch.device(device)
        # Router of this rank's tokens: capacity = T (nothing dropped), weights renormalised if
        # asked; the capacity is applied by the owners.
        self.router = moe.MoELayer(T_local, d_model, d_ff, E, k, math.inf, dtype, device,
                                   flags & moe.FLAG_RENORMALIZE)
        # An owner receives at most min(k, E_local) candidates per token of the whole batch,
        # and keeps at most K of them per expert.
        self.cand_max = max(T_local * world * min(k, E_local), 1)
        self.rows_max = max(min(self.cand_max, E_local * K), 1)
        self.sel_ws = self._ws(self._sel_problem(self.cand_max))
        self.ffn_ws = self._ws(self._ffn_problem(self.rows_max))
        self.comb_ws = torch.zeros(32, dtype=torch.int64, device=self.device)
        self.launches = 0           # kernels this object's calls launched (moe_last_launch_count)

    def _count(self):
        self.launches += moe.moe_last_launch_count()

    def _ws(self, p):
        n = moe.moe_workspace_size(p)
        return torch.zeros((n + 7) // 8, dtype=torch.int64, device=self.device)

    def _sel_problem(self, n):
        return moe.problem(n, 64, 64, self.E_local, 1, math.inf, self.dtype,
                           self.flags & moe.FLAG_ARRIVAL_ORDER)

    def _ffn_problem(self, n):
        return moe.problem(n, self.d_model, self.d_ff, self.E_local, 1, math.inf, self.dtype,
                           self.flags & moe.FLAG_GATED)

    def route(self, x, Wr, br):
        logits = self.router.router_logits(x, Wr, br)
        self._count()
        r = self.router.route(logits)
        self._count()
        return r["ids"], r["w"]

    def select(self, e_v, w_v, K):
        """Capacity selection over the candidates an owner received (k = 1 per candidate)."""
        n = e_v.shape[0]
        dev = e_v.device
        slot = torch.empty((n, 1), dtype=torch.int32, device=dev)
        drop = torch.empty((n, 1), dtype=torch.uint8, device=dev)
        counts = torch.empty(2 * self.E_local, dtype=torch.int32, device=dev)
        offsets = torch.empty(self.E_local + 1, dtype=torch.int32, device=dev)
        rowtok = torch.empty(max(min(n, self.E_local * int(K)), 1), dtype=torch.int32,
                             device=dev)
        moe.moe_capacity_dispatch(self._sel_problem(n), K, e_v.view(n, 1), w_v.view(n, 1), slot,
                                  drop, counts, self.sel_ws, offsets, rowtok)
        self._count()
        return slot.view(n), offsets, rowtok

    def expert_ffn(self, x_rows, offsets, rowtok, W1, b1, W2, b2):
        n = x_rows.shape[0]
        Y = torch.empty((max(n, 1), self.d_model), dtype=x_rows.dtype, device=x_rows.device)
        if n > 0:
            moe.moe_expert_ffn(self._ffn_problem(n), x_rows, offsets, rowtok, W1, b1, W2, b2, Y,
                               self.ffn_ws)
            self._count()
        return Y[:n]

    def combine(self, x, Y_back, w, slot_back):
        """out = x + sum over kept j of w[t, j] Y_back[slot_back[t, j]]: the rows come back in
        one block, addressed as k groups that all start at row 0 and end at its last row."""
        T, k = w.shape
        m = Y_back.shape[0]
        p = moe.problem(T, self.d_model, 64, k, k, math.inf, self.dtype)
        ids = torch.zeros((T, k), dtype=torch.int32, device=x.device)
        offsets = torch.full((k + 1,), m, dtype=torch.int32, device=x.device)
        offsets[0] = 0
        Y = Y_back if m > 0 else torch.zeros((1, self.d_model), dtype=x.dtype, device=x.device)
        out = torch.empty_like(x)
        moe.moe_combine(p, x, Y, w, ids, slot_back, offsets, out, self.comb_ws)
        self._count()
        return out


class ExpertParallelLayer:
    """One MoE layer whose experts are split over the ranks of `group`.

    forward(x, Wr, br, W1, b1, W2, b2): x [T_local, d_model] this rank's tokens; Wr [d_model, E]
    and br [E] the whole router (every rank holds it); W1 [E_local, F, d_model], b1 [E_local, F],
    W2 [E_local, d_model, F], b2 [E_local, d_model] this rank's experts.  Returns out [T_local,
    d_model] and the routing of this rank's tokens: ids, w, slot (the rank among the expert's
    kept tokens of the whole batch, -1 if dropped) and drop.
    """

    def __init__(self, group, T_local, d_model, d_ff, E, k, capacity_factor=math.inf,
                 dtype="bf16", device="cuda", flags=0, steps=None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if E % self.world != 0:
            raise ValueError("E must be a multiple of the number of ranks")
        self.T_local, self.E, self.k = T_local, E, k
        self.E_local = E // self.world
        self.T_global = T_local * self.world
        # The capacity of the whole batch, as the single-device layer computes it.
        self.K = moe.moe_capacity(moe.problem(self.T_global, d_model, d_ff, E, k,
                                              capacity_factor, dtype, flags))
        self.steps = steps if steps is not None else CudaSteps(
            T_local, d_model, d_ff, E, self.E_local, k, self.K, self.world, dtype, device, flags)

    def forward(self, x, Wr, br, W1, b1, W2, b2):
        g, world, k, El = self.group, self.world, self.k, self.E_local
        T = x.shape[0]
        dev = x.device
        ids, w = self.steps.route(x, Wr, br)                          # [T, k] each
        P = T * k
        ids_f = ids.reshape(P).to(torch.int64)
        dest = ids_f // El                                             # owner of each pair
        order, send_cnt = _group_order(dest, world)                    # grouped by owner
        recv_cnt = _a2a_counts(send_cnt, g)
        sc, rc = send_cnt.tolist(), recv_cnt.tolist()
        # Candidates: (local expert, weight), in each source's pair (= token) order.
        e_v = _a2a((ids_f - dest * El)[order].to(torch.int32), sc, rc, g)
        w_v = _a2a(w.reshape(P)[order], sc, rc, g)
        slot_v, offsets, rowtok_v = self.steps.select(e_v, w_v, self.K)
        # Slots back to the sources, in their send order.
        slot_sent = _a2a(slot_v, rc, sc, g)
        slot = torch.empty(P, dtype=torch.int32, device=dev)
        slot[order] = slot_sent
        # x rows of the kept pairs to their owners.  The only host synchronisations of the
        # forward are the two count exchanges; every index below has a size known from them, so
        # no boolean mask is materialised on the host's behalf (nonzero_static).
        kept_sent = slot_sent >= 0
        kcnt_send = torch.zeros(world, dtype=torch.int64, device=dev).scatter_add_(
            0, dest[order], kept_sent.to(torch.int64))
        kcnt_recv = _a2a_counts(kcnt_send, g)
        ks, kr = kcnt_send.tolist(), kcnt_recv.tolist()
        n_sent, n_rows = sum(ks), sum(kr)                              # kept rows sent, received
        at_sent = order[torch.nonzero_static(kept_sent, size=n_sent).view(-1)]
        tok_sent = torch.div(at_sent, k, rounding_mode="floor")
        x_rows = _a2a(x[tok_sent], ks, kr, g)
        # The owner's expert-sorted rows: row offsets[e] + slot holds the kept candidate whose
        # rank among the kept candidates (in arrival order) is the index of its x row.
        kept_v = slot_v >= 0
        kept_rank = torch.cumsum(kept_v.to(torch.int32), 0, dtype=torch.int32) - 1
        rowtok = kept_rank[rowtok_v[:n_rows].to(torch.int64)]
        Y = self.steps.expert_ffn(x_rows, offsets, rowtok, W1, b1, W2, b2)
        # Expert rows back, in the order the x rows came.
        at_v = torch.nonzero_static(kept_v, size=n_rows).view(-1)
        rows_back = offsets[:-1].to(torch.int64)[e_v[at_v].to(torch.int64)] + \
            slot_v[at_v].to(torch.int64)
        Y_back = _a2a(Y[rows_back], kr, ks, g)
        slot_back = torch.full((P,), -1, dtype=torch.int32, device=dev)
        slot_back[at_sent] = torch.arange(n_sent, dtype=torch.int32, device=dev)
        out = self.steps.combine(x, Y_back, w, slot_back.view(T, k))
        slot = slot.view(T, k)
        return out, dict(ids=ids, w=w, slot=slot, drop=(slot < 0).to(torch.uint8))
