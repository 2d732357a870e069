"""Expert parallelism: the layer's routed experts split over G ranks.

superteams.ai "Llama 4" glossary, "Mixture of Experts: Why Total and Active
Parameters Diverge": a token only needs the expert its router picks (and the
shared expert), so the experts can live on different GPUs and the tokens
travel to them.  Rank r of G holds routed experts [r E/G, (r+1) E/G) and a
copy of the shared expert, and feeds its own batch of tokens.  One forward:

  1. route the rank's own T tokens: k entries (expert, gate) per token;
  2. plan the dispatch: each entry goes to the rank holding its expert; the
     entries are sent in (destination, expert, token, slot) order, so every
     destination receives, from each source, its entries grouped by expert;
  3. exchange the per-destination counts (an all-to-all of G integers), then
     the entries' input rows and their (expert, gate) (all-to-alls split by
     those counts);
  4. on each rank, order the received entries by (local expert, source rank,
     position) -- the grouped-GEMM order -- and run each local expert on its
     rows: SwiGLU_e(g * x);
  5. send every result back to its source in the order it was received (the
     reverse all-to-all);
  6. each source adds the returned rows to its tokens' outputs, entry by
     entry in slot order, after the shared expert's output.

This module holds the host-side index arithmetic (steps 2, 4, 5 and 6) and
the exchanges (torch.distributed all-to-alls: NCCL on GPUs, gloo on CPU).
The routing, the expert compute and the shared expert are callables the
caller supplies, so the same plan drives any per-rank compute.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch
import torch.distributed as dist


def experts_of_rank(E: int, G: int, r: int) -> range:
    """The routed experts rank r holds (contiguous, E % G == 0)."""
    if E % G:
        raise ValueError(f"expert parallelism needs E ({E}) divisible by the ranks ({G})")
    n = E // G
    return range(r * n, (r + 1) * n)


@dataclass
class DispatchPlan:
    """Where this rank's entries go.  Entry n = t * k + j is token t's j-th
    selected expert.  order[i] is the entry sent i-th; send_counts[q] entries
    go to rank q (consecutive in `order`)."""
    order: np.ndarray        # int64 [T * k]
    send_counts: np.ndarray  # int64 [G]
    dest: np.ndarray         # int64 [T * k]: destination rank of each entry


def plan_dispatch(idx: np.ndarray, E: int, G: int) -> DispatchPlan:
    """Step 2: idx [T, k] (or [T]) expert of each entry -> the send order,
    stable by (destination, expert, entry)."""
    e = np.asarray(idx, dtype=np.int64).reshape(-1)
    if e.size and (e.min() < 0 or e.max() >= E):
        raise ValueError("expert index out of range")
    per = E // G
    dest = e // per
    # stable sort by expert (destination is a function of the expert, so
    # this is also (destination, expert, entry) order)
    order = np.argsort(e, kind="stable")
    send_counts = np.bincount(dest, minlength=G).astype(np.int64)
    return DispatchPlan(order=order, send_counts=send_counts, dest=dest)


@dataclass
class LocalGroups:
    """Step 4: the received entries in grouped-GEMM order.  order[i] is the
    received position of the i-th entry in that order; counts[e_local] rows
    of each local expert, consecutive."""
    order: np.ndarray   # int64 [n_recv]
    counts: np.ndarray  # int64 [E / G]


def local_groups(recv_expert: np.ndarray, recv_counts: np.ndarray, first_expert: int,
                 n_local: int) -> LocalGroups:
    """Order the received entries by (local expert, source rank, position).
    recv_counts[q] entries came from rank q, in that rank's send order."""
    re = np.asarray(recv_expert, dtype=np.int64) - first_expert
    if re.size and (re.min() < 0 or re.max() >= n_local):
        raise ValueError("received an entry for an expert this rank does not hold")
    # positions are already grouped by source rank (all-to-all layout), so a
    # stable sort by expert keeps (source, position) order inside an expert
    order = np.argsort(re, kind="stable")
    return LocalGroups(order=order, counts=np.bincount(re, minlength=n_local).astype(np.int64))


def _all_to_all(t: torch.Tensor, send_counts, recv_counts, group=None) -> torch.Tensor:
    """Rows of t split by send_counts to the ranks; returns the rows received
    (recv_counts from each rank, in rank order).  16-bit integer rows (bf16
    bit patterns) travel widened to int32 where the backend (gloo) has no
    16-bit all-to-all."""
    narrow = t.dtype == torch.int16 and dist.get_backend(group) == "gloo"
    src = t.to(torch.int32) if narrow else t
    out = torch.empty((int(sum(recv_counts)),) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device)
    dist.all_to_all_single(out, src.contiguous(), output_split_sizes=[int(c) for c in recv_counts],
                           input_split_sizes=[int(c) for c in send_counts], group=group)
    return out.to(torch.int16) if narrow else out


def exchange_counts(send_counts: np.ndarray, device, group=None) -> np.ndarray:
    """Step 3a: every rank learns how many entries each rank sends it."""
    G = len(send_counts)
    s = torch.as_tensor(np.asarray(send_counts, dtype=np.int64), device=device)
    r = torch.empty(G, dtype=torch.int64, device=device)
    dist.all_to_all_single(r, s, group=group)
    return r.cpu().numpy()


def ep_forward(x: torch.Tensor, route, expert, shared, E: int, k: int = 1, group=None) -> torch.Tensor:
    """One expert-parallel forward of this rank's tokens x [T, d].

    route(x) -> (idx [T, k] int, gate [T, k] float): the router's entries.
    expert(e, rows, gates) -> [n, d] float64: expert e (held by this rank) on
      its received rows with their gates (SwiGLU_e(g * x)).
    shared(x) -> [T, d] float64: the shared expert on this rank's tokens.
    Returns out [T, d] float64 = shared + the k routed results in slot order.
    Every rank must call it (the exchanges are collective)."""
    G = dist.get_world_size(group)
    r = dist.get_rank(group)
    T = x.shape[0]
    idx, gate = route(x)
    idx = np.asarray(idx, dtype=np.int64).reshape(T, k)
    gate = np.asarray(gate, dtype=np.float64).reshape(T, k)
    plan = plan_dispatch(idx, E, G)
    recv_counts = exchange_counts(plan.send_counts, x.device, group)
    ent = plan.order
    tok = ent // k
    rows = _all_to_all(x[torch.as_tensor(tok, dtype=torch.long)], plan.send_counts, recv_counts, group)
    meta_e = _all_to_all(torch.as_tensor(idx.reshape(-1)[ent]), plan.send_counts, recv_counts, group)
    meta_g = _all_to_all(torch.as_tensor(gate.reshape(-1)[ent]), plan.send_counts, recv_counts, group)
    mine = experts_of_rank(E, G, r)
    lg = local_groups(meta_e.numpy(), recv_counts, mine.start, len(mine))
    results = torch.zeros((rows.shape[0], x.shape[1]), dtype=torch.float64)
    pos = 0
    for el, n in enumerate(lg.counts):
        sel = lg.order[pos:pos + n]
        pos += n
        if n:
            s = torch.as_tensor(sel, dtype=torch.long)
            results[s] = torch.as_tensor(expert(mine.start + el, rows[s], meta_g[s].numpy()), dtype=torch.float64)
    back = _all_to_all(results, recv_counts, plan.send_counts, group)   # step 5, in send order
    routed = torch.zeros((T * k, x.shape[1]), dtype=torch.float64)
    routed[torch.as_tensor(ent, dtype=torch.long)] = back                # entry order
    out = torch.as_tensor(shared(x), dtype=torch.float64).clone()
    for j in range(k):                                                   # slot order
        out += routed.view(T, k, -1)[:, j]
    return out
