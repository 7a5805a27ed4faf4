"""One rank of the expert-parallel bookkeeping check (run under torch.distributed.run by
tests/test_ep_bookkeeping.py over gloo on CPU; not a test module itself).

Every rank holds a consecutive block of the layer's tokens and routes them with the oracle.  The
token rows travel to the ranks that own their experts with one all_to_all_single, in the order
fp8_fp4_moe_b200.ep.send_plan gives; each receiver regroups them expert-major (recv_plan), runs
the oracle's expert FFN of its local experts, and returns the rows with a second all_to_all
(split sizes swapped).  The sender combines them with its gates in slot order and adds its own
shared-expert row.  Each rank writes what it saw to a file for the test to compare with the
single-device oracle.
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

from fp8_fp4_moe_b200 import ep  # noqa: E402
from fp8_fp4_moe_b200 import inputs as I  # noqa: E402
from oracle import formats as F  # noqa: E402
from oracle import moe as M  # noqa: E402

W = I.Workload("ep", T=64, H=256, I=256, E=16, k=4, shared=1, router_std=0.05, bias="uniform")


def a2a(send: np.ndarray, send_counts, recv_counts, row_elems: int) -> np.ndarray:
    """all_to_all_single of rows (int64 payload so any small integer array travels exactly)."""
    s = torch.from_numpy(np.ascontiguousarray(send, dtype=np.int64).reshape(-1))
    r = torch.empty(int(np.sum(recv_counts)) * row_elems, dtype=torch.int64)
    dist.all_to_all_single(r, s, output_split_sizes=[int(c) * row_elems for c in recv_counts],
                           input_split_sizes=[int(c) * row_elems for c in send_counts])
    return r.numpy().reshape(-1, row_elems) if row_elems > 1 else r.numpy()


def main():
    dist.init_process_group("gloo")
    rank, G = dist.get_rank(), dist.get_world_size()
    try:
        w = W
        layout = ep.EPLayout(w.E, G)
        T_r = w.T // G
        tok0 = rank * T_r
        x, W_r, bias = I.make_routing_inputs(w, 5)
        W1, W1s, W2, W2s = I.make_expert_weights(w, 5)
        W1, W1s, W2, W2s = W1.numpy(), W1s.numpy(), W2.numpy(), W2s.numpy()
        xb = x.view(torch.int16).numpy().view(np.uint16)[tok0:tok0 + T_r]
        ids, gates, _ = M.route(xb, W_r.numpy(), bias.numpy(), w.k)

        # dispatch: counts first (every rank learns what it will receive), then the rows with
        # their (global token, slot) tags
        sp = ep.send_plan(ids, layout)
        seg = a2a(sp.expert_counts, np.full(G, 1), np.full(G, 1), layout.E_loc)     # [G, E_loc]
        rp = ep.recv_plan(seg)
        tok = sp.send_copy // w.k
        send_rows = np.concatenate([xb[tok].astype(np.int64),
                                    (tok0 + tok)[:, None], (sp.send_copy % w.k)[:, None]], axis=1)
        recv = a2a(send_rows, sp.send_counts, rp.recv_counts, w.H + 2)
        recv_x = recv[:, :w.H].astype(np.uint16)

        # local experts on their rows, expert-major; rows returned in arrival order
        out_rows = np.zeros((recv.shape[0], w.H), dtype=np.uint16)
        order = {}
        for l in range(layout.E_loc):
            e = rank * layout.E_loc + l
            rows = rp.group_rows[rp.group_offsets[l]:rp.group_offsets[l + 1]]
            order[str(e)] = recv[rows, w.H].tolist()            # global tokens, expert-major
            if rows.size == 0:
                continue
            xq, xexp = M.quantize_blocks(F.bf16_to_f64(recv_x[rows]))
            res = M.expert_ffn(xq, xexp, W1[e], W1s[e], W2[e], W2s[e], w.I)
            out_rows[rows] = res["row_bits"]
        back = a2a(out_rows.astype(np.int64), rp.recv_counts, sp.send_counts, w.H).astype(np.uint16)

        # combine in slot order, then the locally computed shared expert
        xq, xexp = M.quantize_blocks(F.bf16_to_f64(xb))
        shared = M.expert_ffn(xq, xexp, W1[w.E], W1s[w.E], W2[w.E], W2s[w.E], w.I)
        y = np.zeros((T_r, w.H))
        for j in range(w.k):
            y = y + gates[:, j][:, None] * F.bf16_to_f64(back[sp.send_pos[:, j]])
        y = y + F.bf16_to_f64(shared["row_bits"])
        with open(os.path.join(sys.argv[1], f"ep_rank{rank}.json"), "w") as f:
            json.dump({"rank": rank, "G": G, "T_r": T_r, "ids": ids.tolist(), "y": y.tolist(),
                       "out_bits": F.f64_to_bf16(y).astype(int).tolist(), "order": order,
                       "recv_counts": rp.recv_counts.tolist(), "send_counts": sp.send_counts.tolist(),
                       "returned_tags": [int(v) for v in recv[:, w.H]]}, f)
    finally:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
