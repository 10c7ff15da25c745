"""Expert parallelism across ranks (CPU, world-size-2 gloo process groups).

local_moe_route_b200.ep splits the experts over the ranks: each rank routes
its own tokens, sends every slot's token row to the rank owning the slot's
expert (all-to-all), runs its experts on the rows it received, sends the
outputs back and combines them.  Here the four compute steps are the fp64
oracle (grouping, expert FFN) and plain indexing, so the test checks the
exchange and its index arithmetic: every rank's y must equal the oracle's
single-process layer for its tokens, and every rank must receive exactly the
slots routed to its experts."""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """The EP compute steps on the CPU in fp64 (test stand-ins for the CUDA
    library): grouping by the oracle's stable counting sort, each expert's
    SwiGLU FFN by the oracle's layer with the route given, the combine as the
    layer's definition."""

    def __init__(self, inp, group_size, El):
        self.inp, self.G, self.El = inp, group_size, El

    def group(self, keys, nkeys):
        import oracle
        ids = keys.numpy().astype(np.int32).reshape(-1, 1)
        counts, offsets, order, pos = oracle.permute(ids, nkeys)
        t = lambda a: torch.from_numpy(np.asarray(a, np.int32))
        return t(counts), t(offsets), t(order), t(pos)

    def gather(self, src, index):
        return src[index.long()]

    def ffn(self, rows, order, offsets, rank):
        import oracle
        from moe_inputs import bf16_bits
        R = rows.shape[0]
        seg = np.searchsorted(offsets.numpy(), np.arange(R), side="right") - 1
        experts = (rank * self.El + seg).astype(np.int32).reshape(R, 1)
        # the received rows hold bf16 values exactly: their bit patterns
        xb = bf16_bits(rows[order.long()].numpy().astype(np.float32))
        tmp = dict(self.inp, x=xb, bias=None)
        res = oracle.moe_forward(tmp, 1, self.G, ids=experts, w=np.ones((R, 1)))
        return torch.from_numpy(res["y"])

    def combine(self, rows, w, position, T, k):
        r = rows.numpy()[position.long().numpy()].reshape(T, k, -1)
        return torch.from_numpy(np.einsum("tk,tkd->td", w.numpy(), r))


def _worker(rank, world, port, bias_hot, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from local_moe_route_b200.ep import ExpertParallelMoE, owner_of
        from moe_inputs import make_custom
        T, d, E, k, n, G = 24, 256, 8, 2, 128, 64
        inp = make_custom(T=T, d=d, E=E, k=k, n=n, group=G, seed=77)
        if bias_hot:
            # every token routes to experts 0 and 1: rank 1 receives nothing
            b = np.zeros(E, np.float32)
            b[[0, 1]] = 100.0
            inp["bias"] = b
        lg = oracle.router_logits(inp["x"], inp["w_router"], inp.get("bias"))
        ids, w = oracle.topk_softmax(lg, k)
        mine = np.arange(rank * T // world, (rank + 1) * T // world)
        x = torch.from_numpy((inp["x"][mine].astype(np.uint32) << 16).view(np.float32)
                             .astype(np.float64))
        ep = ExpertParallelMoE(E, k, OracleOps(inp, G, E // world))
        stats = {}
        y = ep.forward(x, torch.from_numpy(ids[mine]), torch.from_numpy(w[mine]), stats)
        ref = oracle.moe_forward(inp, k, G, tokens=mine)["y"]
        err = float(np.max(np.abs(y.numpy() - ref)) / np.sqrt(np.mean(ref ** 2)))
        owners = owner_of(torch.from_numpy(ids), E, world).numpy()
        expect_recv = int(np.sum(owners == rank))
        sent = [int(np.sum(owners[mine] == r)) for r in range(world)]
        q.put((rank, err, sum(stats["received"]), expect_recv, stats["sent"], sent))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("bias_hot", [False, True], ids=["uniform", "one_rank_idle"])
def test_expert_parallel_forward_matches_single_process_oracle(bias_hot):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, bias_hot, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, err, recv, expect_recv, sent, expect_sent in res:
        assert err <= 1e-12, (rank, err)
        assert recv == expect_recv and sent == expect_sent, (rank, recv, expect_recv)
    if bias_hot:
        assert res[1][2] == 0          # the second rank owns no chosen expert


def test_expert_split_rules():
    sys.path.insert(0, ROOT)
    from local_moe_route_b200.ep import experts_per_rank, owner_of
    assert experts_per_rank(512, 8) == 64
    with pytest.raises(ValueError):
        experts_per_rank(10, 4)
    assert owner_of(torch.tensor([0, 63, 64, 511]), 512, 8).tolist() == [0, 0, 1, 7]
