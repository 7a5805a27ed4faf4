"""Index bookkeeping of the expert-parallel layer (experts sharded over G ranks).

The pages' design ("Mega MoE" wiki, "어떻게 작동하나"; "DeepSeek Mega MoE / DeepGEMM mega
kernel", "Có gì mới" and "Thông số kỹ thuật": expert parallelism over NVLink, EP <= 8) shards
the routed experts over the GPUs and moves token copies to the GPU that owns their expert
(dispatch) and the expert rows back (combine).  This module fixes WHICH rows go WHERE and in
WHICH order -- no arithmetic of the layer, no data movement; the exchange itself is one
all-to-all per direction with the split sizes given here (NCCL between GPUs, gloo in the CPU
tests).

Layout:
  * routed expert e lives on rank e // E_loc (E_loc = E / G experts per rank, contiguous
    blocks), as local expert e % E_loc; the shared expert is replicated on every rank and
    never leaves it;
  * every rank holds T_r tokens and routes them itself (the router weights are replicated);
  * send order of a rank = its single-device dispatch order (expert-major, ascending token
    inside an expert): because each rank owns a contiguous block of experts, that order is
    already grouped by destination rank, so the send buffer is the dispatched-row buffer and
    the split sizes are sums of per-expert counts;
  * rows arrive grouped by source rank (rank order) and, inside a source's chunk, expert-major;
    a receiver regroups them expert-major with sources in rank order.  When the ranks hold
    consecutive blocks of global token ids (rank r holds tokens r*T_r ...), this receive order
    of expert e is exactly the single-device dispatch order of expert e (ascending global
    token), so the expert FFN sees the same rows in the same order on one device and on G;
  * combine: each receiver returns the expert rows in the order the rows arrived (the reverse
    all-to-all with the split sizes swapped), so a sender finds the row of its copy (t, j) at
    its send position, exactly where the single-device combine reads it.
"""
from __future__ import annotations

import dataclasses

import numpy as np

__all__ = ["EPLayout", "SendPlan", "RecvPlan", "send_plan", "recv_plan"]


@dataclasses.dataclass(frozen=True)
class EPLayout:
    E: int          # routed experts
    G: int          # ranks

    def __post_init__(self):
        if self.G < 1 or self.E % self.G != 0:
            raise ValueError(f"E = {self.E} routed experts do not split evenly over G = {self.G} ranks")

    @property
    def E_loc(self) -> int:
        return self.E // self.G

    def owner(self, e):
        return np.asarray(e) // self.E_loc

    def local(self, e):
        return np.asarray(e) % self.E_loc


@dataclasses.dataclass
class SendPlan:
    """What one rank sends.  copy (t, j) = token t's j-th selected expert, copy id t*k + j."""
    send_copy: np.ndarray        # [T_r * k] copy ids in send order
    send_pos: np.ndarray         # [T_r, k] send position of copy (t, j)
    send_counts: np.ndarray      # [G] rows to each destination rank
    expert_counts: np.ndarray    # [G, E_loc] rows to each (destination, its local expert)


@dataclasses.dataclass
class RecvPlan:
    """What one rank receives, from the G ranks' expert_counts[:, this rank] rows."""
    recv_counts: np.ndarray      # [G] rows from each source rank (source order)
    seg_counts: np.ndarray       # [G, E_loc] rows from source s for local expert l
    group_rows: np.ndarray       # [R_in] arrival index of each row in expert-major order (l, s, t)
    group_counts: np.ndarray     # [E_loc] rows per local expert
    group_offsets: np.ndarray    # [E_loc + 1]


def send_plan(topk_ids: np.ndarray, layout: EPLayout) -> SendPlan:
    """Send order of a rank's copies: expert-major, ascending token inside an expert."""
    ids = np.asarray(topk_ids, dtype=np.int64)
    T, k = ids.shape
    if ids.size and (ids.min() < 0 or ids.max() >= layout.E):
        raise ValueError("expert id out of range")
    copy = np.arange(T * k, dtype=np.int64)
    e = ids.reshape(-1)
    tok = copy // k
    order = np.lexsort((tok, e))                         # primary: expert; secondary: token
    send_copy = copy[order]
    send_pos = np.empty(T * k, dtype=np.int64)
    send_pos[send_copy] = np.arange(T * k, dtype=np.int64)
    per_expert = np.bincount(e, minlength=layout.E)
    expert_counts = per_expert.reshape(layout.G, layout.E_loc)
    return SendPlan(send_copy=send_copy, send_pos=send_pos.reshape(T, k),
                    send_counts=expert_counts.sum(axis=1), expert_counts=expert_counts)


def recv_plan(seg_counts: np.ndarray) -> RecvPlan:
    """seg_counts[s, l]: rows source rank s sends for this rank's local expert l (its
    SendPlan.expert_counts[this rank], gathered).  Rows arrive source after source, each
    source's rows expert-major; group_rows lists them expert-major with sources in order."""
    seg = np.asarray(seg_counts, dtype=np.int64)
    G, E_loc = seg.shape
    recv_counts = seg.sum(axis=1)
    src_base = np.concatenate([[0], np.cumsum(recv_counts)])
    seg_base = src_base[:-1, None] + np.concatenate([np.zeros((G, 1), np.int64), np.cumsum(seg, axis=1)[:, :-1]],
                                                    axis=1)
    group_rows = [np.arange(seg_base[s, l], seg_base[s, l] + seg[s, l]) for l in range(E_loc) for s in range(G)]
    group_rows = np.concatenate(group_rows) if group_rows else np.zeros(0, np.int64)
    group_counts = seg.sum(axis=0)
    return RecvPlan(recv_counts=recv_counts, seg_counts=seg, group_rows=group_rows.astype(np.int64),
                    group_counts=group_counts, group_offsets=np.concatenate([[0], np.cumsum(group_counts)]))
