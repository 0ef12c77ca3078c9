"""Expert-parallel dispatch / combine index math on two gloo ranks (CPU).

Each rank routes its own tokens with the oracle's router, sends the rows of
its compact expert-sorted order to the rank that owns their experts, and gets
them back after an identity "expert computation".  Checked: every received
row lands in its local expert's span of the aligned row space, rows inside a
span are ordered by (source rank, token, slot), spans are 128-aligned, and
every slot receives its own row back at its compact position."""
import json
import os
import socket

import numpy as np
import pytest


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir, E, k):
    import datetime

    import torch
    import torch.distributed as dist

    import oracle as O
    import synthetic as S
    from grouped_gemm_moesq_b200 import ep
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        T = 37 + 11 * rank                                     # ranks hold different token counts
        lg = S.zipf_logits_np(100 + rank, T, E)
        rt = O.route(lg, k)
        El = ep.experts_per_rank(E, world)
        send_counts, per_expert = ep.send_plan(rt.offsets, world)
        from_src = ep.exchange_counts(per_expert)
        recv_counts = from_src.sum(axis=1)
        # payload: (source rank, slot, expert) of every row of the compact order
        slots = rt.sorted_to_slot.astype(np.int64)
        experts = rt.expert_of_sorted().astype(np.int64)
        payload = torch.as_tensor(np.stack([np.full_like(slots, rank), slots, experts], axis=1))
        got = ep.exchange_rows(payload, send_counts, recv_counts).numpy()
        counts, row_offsets, dest = ep.recv_layout(from_src)
        # identity expert computation in the aligned row space, then gather back
        space = np.full((int(row_offsets[-1]), 3), -1, np.int64)
        space[dest] = got
        back = torch.as_tensor(space[dest])
        ret = ep.exchange_rows(back, recv_counts, send_counts).numpy()
        res = {"rank": rank, "T": T, "El": El, "counts": counts.tolist(), "row_offsets": row_offsets.tolist(),
               "space": space.tolist(), "ret": ret.tolist(), "slots": slots.tolist(), "experts": experts.tolist(),
               "slot_to_sorted": rt.slot_to_sorted.tolist(), "k": k}
        dist.barrier()
        with open(os.path.join(out_dir, "ep%d.json" % rank), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("E,k", [(8, 2), (16, 4)])
def test_ep_dispatch_and_combine_two_ranks(tmp_path, E, k):
    mp = pytest.importorskip("torch.multiprocessing")
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path), E, k), nprocs=world, join=True)
    r = [json.load(open(tmp_path / ("ep%d.json" % i))) for i in range(world)]
    El = E // world
    for d in range(world):
        space = np.array(r[d]["space"])
        ro = np.array(r[d]["row_offsets"])
        assert (ro % 128 == 0).all()
        for e in range(El):
            span = space[ro[e]:ro[e + 1]]
            rows = span[span[:, 0] >= 0]
            assert len(rows) == r[d]["counts"][e]
            assert (rows[:, 2] == d * El + e).all()                      # only this expert's rows
            assert (span[len(rows):, 0] == -1).all()                      # padding after the rows
            key = [(int(a), int(b)) for a, b, _ in rows]
            assert key == sorted(key)                                     # source, then token, then slot
            # every row routed to this expert by any source arrives
            want = sorted((s, slot) for s in range(world)
                          for slot, ex in zip(r[s]["slots"], r[s]["experts"]) if ex == d * El + e)
            assert key == want
    for s in range(world):
        ret = np.array(r[s]["ret"])
        # row i of the return is the sender's compact position i: its own row back
        assert (ret[:, 0] == s).all()
        assert (ret[:, 1] == np.array(r[s]["slots"])).all()
        # the combine finds slot (t, j) at its compact position
        s2s = np.array(r[s]["slot_to_sorted"])
        assert (ret[s2s, 1] == np.arange(r[s]["T"] * r[s]["k"])).all()


def test_send_plan_and_layout_single_process():
    from grouped_gemm_moesq_b200 import ep
    offsets = np.array([0, 3, 3, 10, 12, 20, 21, 21, 30])
    send, per = ep.send_plan(offsets, 2)
    assert send.tolist() == [12, 18] and per.tolist() == [[3, 0, 7, 2], [8, 1, 0, 9]]
    counts, ro, dest = ep.recv_layout(np.array([[3, 0, 7, 2], [1, 129, 0, 0]]))
    assert counts.tolist() == [4, 129, 7, 2] and ro.tolist() == [0, 128, 384, 512, 640]
    assert dest[:3].tolist() == [0, 1, 2] and dest[3:10].tolist() == list(range(384, 391))
    assert dest[12] == 3 and dest[13:].tolist() == list(range(128, 257))
    with pytest.raises(ValueError):
        ep.experts_per_rank(10, 4)
