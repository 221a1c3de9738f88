"""Expert parallelism for the routed-experts layer (the dispatch / combine of
the DeepGEMM Mega MoE news page and of the "MegaMOE adaptation for SM90" PR,
without their fused kernels).

The E experts are sharded over the ranks of a group: rank r owns experts
[r*E/G, (r+1)*E/G).  Every rank holds its own tokens and their routing.  One
forward:

  1. plan      the valid slots (t, k) of this rank, ordered by the owner rank
               of their expert (slots in ascending order inside one owner):
               the same stable order as the permutation step of the
               single-GPU path, coarsened to ranks;
  2. dispatch  all-to-all of the slots' hidden rows, local expert ids and
               router weights to the owners;
  3. experts   the owner runs its received rows through moe_experts_rows
               (grouped GEMMs, one slot per row): y = w * expert(x), fp32;
  4. return    all-to-all of the y rows back, in the order they were sent;
  5. combine   moe_combine_rows sums each token's K rows in k order (fixed
               order, no atomics) and rounds once to bf16.

Because every row is computed by the same kernels and summed in the same
order as on one GPU, the result does not depend on how the experts are
sharded.  The data plane is torch.distributed's all_to_all_single (NCCL over
NVLink on GPUs, gloo on CPU); no load of another GPU's memory is made by the
library's kernels, so no cluster-multicast load ever reads peer memory.
"""
from typing import Callable, Optional

import torch


def experts_per_rank(E: int, world: int) -> int:
    if world < 1 or E % world:
        raise ValueError("E (%d) must be a multiple of the group size (%d)" % (E, world))
    return E // world


def ep_plan(top_k_index: torch.Tensor, E: int, world: int):
    """Dispatch plan of this rank's slots.

    Returns (order, send_counts, local_ids):
      order       int64 [n_send]: slot indices t*K+k of the valid slots, by
                  owner rank, ascending inside one owner;
      send_counts int64 [world]: slots sent to each rank;
      local_ids   int32 [n_send]: the slot's expert id on its owner rank.
    Slots whose id is outside [0, E) are not sent (they contribute nothing).
    """
    El = experts_per_rank(E, world)
    flat = top_k_index.reshape(-1).to(torch.int64)
    valid = (flat >= 0) & (flat < E)
    owner = torch.where(valid, flat // El, torch.full_like(flat, world))
    order = torch.sort(owner, stable=True).indices
    n_send = int(valid.sum().item())
    order = order[:n_send]
    send_counts = torch.bincount(owner[valid], minlength=world)[:world]
    local_ids = (flat[order] - owner[order] * El).to(torch.int32)
    return order, send_counts, local_ids


class TorchDistExchange:
    """The all-to-all of a torch.distributed group (NCCL or gloo)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def counts(self, send_counts: torch.Tensor) -> torch.Tensor:
        recv = torch.empty_like(send_counts)
        self.dist.all_to_all_single(recv, send_counts, group=self.group)
        return recv

    def rows(self, send: torch.Tensor, send_splits, recv_splits) -> torch.Tensor:
        """send [n, ...] split by send_splits -> [sum(recv_splits), ...]."""
        recv = torch.empty((sum(recv_splits),) + tuple(send.shape[1:]), dtype=send.dtype,
                           device=send.device)
        self.dist.all_to_all_single(recv, send, recv_splits, send_splits, group=self.group)
        return recv


def _as_words(t: torch.Tensor) -> torch.Tensor:
    """16-bit rows as int32 words for the transport (gloo has no 16-bit types)."""
    return t.view(torch.int32) if t.element_size() == 2 else t


def ep_forward(hidden_states: torch.Tensor, gate_up_local: torch.Tensor, down_local: torch.Tensor,
               top_k_index: torch.Tensor, top_k_weights: torch.Tensor, E: int,
               exchange=None, rows_fn: Optional[Callable] = None,
               combine_fn: Optional[Callable] = None) -> torch.Tensor:
    """Routed-experts forward with the experts sharded over the exchange's
    ranks: gate_up_local [E/G, 2F, H] and down_local [E/G, H, F] are this
    rank's experts (global ids rank*E/G ...).  Returns out [T, H] bf16 for
    this rank's tokens.

    rows_fn(x [R,H] bf16, ids [R,1] int32, w [R,1] fp32) -> y [R,H] fp32 and
    combine_fn(y [T*K,H] fp32, top_k_index) -> out default to the library's
    moe_experts_rows / moe_combine_rows."""
    from . import moe_combine_rows, moe_experts_rows
    ex = exchange if exchange is not None else TorchDistExchange()
    T, K = top_k_index.shape
    H = hidden_states.shape[1]
    order, send_counts, local_ids = ep_plan(top_k_index, E, ex.world)
    if rows_fn is None:
        def rows_fn(xr, ir, wr):
            return moe_experts_rows(xr, gate_up_local, down_local, ir, wr, 1).clone()
    if combine_fn is None:
        def combine_fn(y, idx):
            return moe_combine_rows(y, idx, E)
    # dispatch: rows, local ids and weights of the sent slots, by owner
    x_send = hidden_states.index_select(0, order // K).contiguous()
    w_send = top_k_weights.reshape(-1).index_select(0, order).contiguous()
    recv_counts = ex.counts(send_counts)
    s_split = [int(c) for c in send_counts.tolist()]
    r_split = [int(c) for c in recv_counts.tolist()]
    x_recv = ex.rows(_as_words(x_send), s_split, r_split).view(hidden_states.dtype).view(-1, H)
    ids_recv = ex.rows(local_ids.contiguous(), s_split, r_split)
    w_recv = ex.rows(w_send, s_split, r_split)
    # this rank's experts on the rows it received
    y_recv = rows_fn(x_recv, ids_recv.view(-1, 1).contiguous(), w_recv.view(-1, 1).contiguous())
    # return and combine
    y_back = ex.rows(y_recv.contiguous(), r_split, s_split)
    y = torch.zeros(T * K, H, dtype=torch.float32, device=hidden_states.device)
    y.index_copy_(0, order, y_back)
    return combine_fn(y, top_k_index)
