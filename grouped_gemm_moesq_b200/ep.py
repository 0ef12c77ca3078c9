"""Expert-parallel split of the MoE layer over G ranks: the dispatch and
combine index plan and the NCCL exchanges (the paper serves with data
parallelism across GPUs and expert parallelism for the routed experts,
App. D.3, where DeepEP's all-to-all moves the tokens).

Rank g owns the experts [g*El, (g+1)*El), El = E / G, and routes its own T
tokens (moesq_route_permute).  Its compact expert-sorted order (offsets)
already groups the slots by destination rank, because every rank's experts
are contiguous, so:

* dispatch: rank g sends, to every rank d, the rows of its compact order
  that belong to d's experts -- send_counts[d] = offsets[(d+1)*El] -
  offsets[d*El] rows, as NVFP4 codes (K/2 bytes) and row-major UE4M3 scales
  (K/32 bytes): 0.5625 bytes per element, quantised at the source with the
  expert's static global scale.  A first exchange of the [G, El] per-expert
  count matrix tells every receiver how many rows of each of its experts
  each source sends.
* receive layout: rank d stacks, for each local expert, the rows of source
  0, then source 1, ..., each 128-row aligned expert span starting at
  row_offsets[e] (the grouped GEMM's expert-aligned row space), and runs the
  local part of the layer (gate_up, SwiGLU + requantise, down) on it.
* combine: the bf16 down-projection rows travel back by the inverse
  exchange, arriving in the sender's compact order, and the router-weighted
  combine reads slot (t, j) at its compact position.

The exchanges are NCCL all-to-all-v calls over NVLink 5 / NVSwitch (uniform
bandwidth to every peer): plain loads and stores, no TMA multicast of any
kind, remote rows land in local memory before a kernel reads them.  This
module holds the host-side index math (numpy) and the exchange calls; the
tests run both on gloo ranks on the CPU.
"""
from __future__ import annotations

import numpy as np

ROW_ALIGN = 128


def experts_per_rank(E: int, G: int) -> int:
    if E % G:
        raise ValueError("experts (%d) must split evenly over %d ranks" % (E, G))
    return E // G


def send_plan(offsets: np.ndarray, G: int):
    """Compact expert offsets [E+1] of this rank's routing -> (send_counts [G]
    rows to each rank, per_expert [G, El] rows of each destination expert),
    both int64."""
    offsets = np.asarray(offsets, np.int64)
    E = offsets.size - 1
    El = experts_per_rank(E, G)
    counts = np.diff(offsets)
    per_expert = counts.reshape(G, El)
    return per_expert.sum(axis=1), per_expert


def recv_layout(from_src: np.ndarray, align: int = ROW_ALIGN):
    """Rows of each local expert from each source, [G, El] (row s of the
    matrix is what source s sends), -> (counts [El], row_offsets [El+1] of
    the aligned row space, dest [R_recv]: the aligned row of every received
    row, in arrival order: source-major, then local expert, then the
    source's compact order)."""
    from_src = np.asarray(from_src, np.int64)
    G, El = from_src.shape
    counts = from_src.sum(axis=0)
    spans = (counts + align - 1) // align * align
    row_offsets = np.concatenate([[0], np.cumsum(spans)]).astype(np.int64)
    # start of source s's rows inside expert e's span: rows of sources < s
    within = np.concatenate([np.zeros((1, El), np.int64), np.cumsum(from_src, axis=0)[:-1]], axis=0)
    dest = []
    for s in range(G):
        for e in range(El):
            n = int(from_src[s, e])
            base = row_offsets[e] + within[s, e]
            dest.append(base + np.arange(n, dtype=np.int64))
    dest = np.concatenate(dest) if dest else np.zeros(0, np.int64)
    return counts, row_offsets, dest


def exchange_rows(rows, send_counts, recv_counts, group=None):
    """All-to-all-v of rows (a torch tensor [R_send, ...] in destination-rank
    order) -> [R_recv, ...] in source-rank order."""
    import torch
    import torch.distributed as dist
    out = torch.empty((int(np.sum(recv_counts)),) + tuple(rows.shape[1:]), dtype=rows.dtype, device=rows.device)
    dist.all_to_all_single(out, rows.contiguous(), [int(c) for c in recv_counts], [int(c) for c in send_counts],
                           group=group)
    return out


def exchange_counts(per_expert: np.ndarray, group=None, device="cpu"):
    """Every rank's [G, El] send matrix -> this rank's [G, El] receive matrix
    (row s: the rows of each local expert that source s sends)."""
    import torch
    import torch.distributed as dist
    G, El = per_expert.shape
    inp = torch.as_tensor(np.ascontiguousarray(per_expert, np.int64), device=device).reshape(G * El)
    out = torch.empty(G * El, dtype=torch.int64, device=device)
    dist.all_to_all_single(out, inp, [El] * G, [El] * G, group=group)
    return out.cpu().numpy().reshape(G, El)
