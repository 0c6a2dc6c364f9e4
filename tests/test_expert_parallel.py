"""Expert parallelism: the exchange layout on the host, across processes, and
the whole layer with its experts split over ranks emulated on one GPU.

"Expert Parallelism: MoE 模型的并行切分" sections 3 and 8, "LLM MoE Expert
Parallel 生产实战" steps 2 and 4: rank r owns experts [r E/n, (r+1) E/n);
each rank sends its kept rows to the experts' owners and gets the results
back.

CPU (no GPU):
  - moe_ep_plan_host on random counts: every (source, expert, row) of the
    exchange lands on exactly one received row, the sender's send base and the
    receiver's layout agree, and every received row returns to the row of the
    source's own dispatch layout it came from;
  - two gloo ranks, each with its own counts: after an all-gather of the
    counts each computes its plan, the rows each rank "sends" (row ids, moved
    with an all-gather) fill every receiver's buffer exactly as its plan says.
GPU (one B200): n ranks' tokens, routing, exchange buffers and experts in
one device's memory; the dispatch and return kernels store into the
destination rank's buffers, each rank runs its experts on what it received,
and every rank's output matches the oracle on its own tokens.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from routing_dispatch_expert_sigmoid_b200 import ops  # noqa: E402
from routing_dispatch_expert_sigmoid_b200.workloads import WORKLOADS, make_inputs  # noqa: E402


def _check_plan(C, n, rank):
    """The layout invariants of one rank's plan (host mirror)."""
    E = C.shape[1]
    e_loc = E // n
    R = int(C[:, rank * e_loc:(rank + 1) * e_loc].sum())
    ro, sb, src, srow = ops.moe_ep_plan_host(n, E, rank, C, R)
    assert ro[0] == 0 and ro[-1] == R and (np.diff(ro) >= 0).all()
    for j in range(e_loc):  # expert sizes: rows of all sources
        assert ro[j + 1] - ro[j] == C[:, rank * e_loc + j].sum()
    # a received row per (source, expert, index), in (expert, source, index) order
    expect_src, expect_row = [], []
    for j in range(e_loc):
        e = rank * e_loc + j
        for s in range(n):
            first = int(C[s, :e].sum())
            expect_src += [s] * int(C[s, e])
            expect_row += list(range(first, first + int(C[s, e])))
    assert (src == np.array(expect_src, np.int32)).all()
    assert (srow == np.array(expect_row, np.int32)).all()
    return ro, sb, src, srow


@pytest.mark.parametrize("n,E", [(1, 8), (2, 8), (4, 64), (8, 256), (8, 1024)])
def test_plan_layout_is_a_bijection(n, E):
    rng = np.random.default_rng(n * 1000 + E)
    C = rng.integers(0, 40, size=(n, E)).astype(np.int32)
    C[rng.random((n, E)) < 0.2] = 0  # some empty (source, expert) pairs
    plans = [_check_plan(C, n, r) for r in range(n)]
    e_loc = E // n
    # the senders' view: row i of source s for expert e lands at send_base_s[e] + i
    # of the owner, which the owner's layout maps back to (s, its row)
    for s in range(n):
        sb = plans[s][1]
        for e in range(E):
            owner = e // e_loc
            _, _, src, srow = plans[owner]
            first = int(C[s, :e].sum())
            for i in range(int(C[s, e])):
                p = sb[e] + i
                assert src[p] == s and srow[p] == first + i


def test_plan_rejects_bad_arguments():
    C = np.zeros((2, 8), np.int32)
    with pytest.raises(ops.MoeError):
        ops.moe_ep_plan_host(3, 8, 0, np.zeros((3, 8), np.int32), 0)  # 3 does not divide 8
    with pytest.raises(ops.MoeError):
        ops.moe_ep_plan_host(2, 8, 2, C, 0)  # no rank 2
    C[1, 0] = 5
    with pytest.raises(ops.MoeError):
        ops.moe_ep_plan_host(2, 8, 0, C, 4)  # 5 received rows do not fit 4


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, n, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=n)
    try:
        E = 16
        rng = np.random.default_rng(100 + rank)
        counts = torch.from_numpy(rng.integers(0, 7, size=E).astype(np.int32))
        gathered = [torch.zeros(E, dtype=torch.int32) for _ in range(n)]
        dist.all_gather(gathered, counts)  # the counts exchange every rank needs first
        C = torch.stack(gathered).numpy()
        R_local = int(C[rank].sum())
        e_loc = E // n
        R_recv = int(C[:, rank * e_loc:(rank + 1) * e_loc].sum())
        ro, sb, src, srow = ops.moe_ep_plan_host(n, E, rank, C, R_recv)
        # this rank's "rows": (rank, row) ids in its own layout, expert-major
        row_expert = np.repeat(np.arange(E), C[rank])
        idx_in_e = np.concatenate([np.arange(c) for c in C[rank]]) if R_local else np.zeros(0, int)
        sends = np.stack([row_expert // e_loc, sb[row_expert] + idx_in_e,
                          np.full(R_local, rank), np.arange(R_local)], axis=1).astype(np.int64)
        # move every rank's sends to everybody (the transport of a real
        # all-to-all is NVLink stores; here the gloo all-gather of the ids)
        sizes = [torch.zeros(1, dtype=torch.int64) for _ in range(n)]
        dist.all_gather(sizes, torch.tensor([R_local], dtype=torch.int64))
        width = int(max(s.item() for s in sizes))
        buf = torch.full((width, 4), -1, dtype=torch.int64)
        buf[:R_local] = torch.from_numpy(sends)
        alls = [torch.zeros_like(buf) for _ in range(n)]
        dist.all_gather(alls, buf)
        received = np.full((R_recv, 2), -1, np.int64)
        for t in alls:
            for owner, pos, s_rank, s_row in t.numpy():
                if owner == rank:
                    assert received[pos, 0] == -1, "two rows for one slot"
                    received[pos] = (s_rank, s_row)
        ok = bool((received[:, 0] == src).all() and (received[:, 1] == srow).all())
        q.put((rank, ok, R_recv))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_exchange():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(ok for _, ok, _ in res), res


# ---------------------------------------------------------------------------
# GPU: n ranks emulated on one device
# ---------------------------------------------------------------------------
EP_CASES = {
    "mixtral_2ranks": (WORKLOADS["mixtral_prefill"].scaled(T=96, d=256, f=384), 2),
    "mixtral_4ranks_decode": (WORKLOADS["mixtral_decode"].scaled(T=24, d=512, f=256), 4),
    "qwen3_4ranks_drops": (WORKLOADS["qwen3_prefill"].scaled(T=200, d=192, E=16, k_max=4,
                                                             f=200), 4),
    "dsv3_8ranks": (WORKLOADS["dsv3_prefill"].scaled(T=64, d=256, E=64, f=136, f_shared=0), 8),
    "gptoss_2ranks_variable_k": (WORKLOADS["gptoss_sub"].scaled(T=120, d=200, E=32, k_max=6,
                                                                k_min=2, f=72), 2),
}


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(EP_CASES))
def test_expert_parallel_layer_emulated_on_one_gpu(name, cuda_device):
    import oracle
    from parity import assert_out_close, check_routing_bit_exact, f64, oracle_layer_on_tokens, \
        run_route, storage
    dev = cuda_device
    w, n = EP_CASES[name]
    E, k, T, d = w.E, w.k_max, w.T, w.d
    e_loc = E // n
    # one set of experts; every rank its own tokens (seed = rank)
    ranks = []
    base = make_inputs(w, seed=0, device=dev)
    for r in range(n):
        own = make_inputs(w, seed=100 + r, device=dev)
        inp = dict(base, x=own["x"], k_per_token=own["k_per_token"])
        cfg, rb = run_route(w, inp)
        routing = check_routing_bit_exact(w, inp, rb)
        ranks.append(dict(inp=inp, cfg=cfg, rb=rb, routing=routing))
    C = torch.stack([rk["rb"]["kept"] for rk in ranks]).contiguous()  # the gathered counts
    rows_cap = T * k
    recv = [torch.zeros((n * rows_cap, d), dtype=base["x"].dtype, device=dev) for _ in range(n)]
    yback = [torch.full((rows_cap, d), float("nan"), dtype=torch.float32, device=dev)
             for _ in range(n)]
    eps = [ops.ep_ranks(r, n, C, recv, yback) for r in range(n)]
    plans = []
    for r, rk in enumerate(ranks):
        ro = torch.empty(e_loc + 1, dtype=torch.int32, device=dev)
        sb = torch.empty(E, dtype=torch.int32, device=dev)
        ops.moe_ep_plan(rk["cfg"], eps[r], ro, sb)
        plans.append((ro, sb))
    for r, rk in enumerate(ranks):  # dispatch: every rank stores into the owners' buffers
        rb = rk["rb"]
        ops.moe_ep_dispatch(rk["cfg"], eps[r], rk["inp"]["x"], rb["offsets"], rb["row_src"],
                            rb["topk_idx"], plans[r][1])
    ops.moe_check_errors()
    Ch = C.cpu().numpy()
    for r in range(n):  # the received rows are the plan's rows, bit for bit
        ro_h, sb_h, src, srow = ops.moe_ep_plan_host(n, E, r, Ch, n * rows_cap)
        assert (plans[r][0].cpu().numpy() == ro_h).all() and (plans[r][1].cpu().numpy() == sb_h).all()
        R = int(ro_h[-1])
        want = torch.stack([ranks[s]["inp"]["x"][int(ranks[s]["routing"]["row_src"][row]) // k]
                            for s, row in zip(src, srow)]) if R else recv[r][:0]
        assert torch.equal(recv[r][:R], want), f"rank {r}: received rows"
    y_recv = []
    for r in range(n):  # each rank: its experts on what it received
        # the FFN over this rank's e_loc experts and up to n * T * k received rows
        # (the gating fields play no part in the FFN)
        wl = w.scaled(E=e_loc, T=n * T, gating="topk_softmax", n_groups=1, topk_groups=1,
                      group_score_topk=1)
        cfg_l = ops.config(wl)
        sl = slice(r * e_loc, (r + 1) * e_loc)
        y = torch.zeros((n * rows_cap, d), dtype=torch.float32, device=dev)
        ops.moe_expert_ffn(cfg_l, recv[r], plans[r][0], base["W1"][sl].contiguous(),
                           base["W3"][sl].contiguous(), base["W2"][sl].contiguous(), y,
                           ops.workspace(cfg_l, ops.WS_EXPERT_FFN))
        y_recv.append(y)
    for r, rk in enumerate(ranks):  # return: every rank stores into the sources' buffers
        ops.moe_ep_return(rk["cfg"], eps[r], y_recv[r], plans[r][0])
    ops.moe_check_errors()
    for r, rk in enumerate(ranks):  # combine on each rank, against the oracle
        out = torch.empty_like(rk["inp"]["x"])
        rb = rk["rb"]
        ops.moe_combine(rk["cfg"], yback[r], rb["slot_row"], rb["topk_w"], None, out)
        ops.moe_check_errors()
        ref = oracle_layer_on_tokens(rk["inp"], rk["routing"], list(range(T)))
        assert_out_close(f64(out), ref, f"{name} rank {r} of {n}", storage(w))
