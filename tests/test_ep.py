"""Expert-parallel form of the block (include/srm_ep.h, sigmoid_routed_mixture_b200/ep.py).

CPU: the partition, the host plan against a brute-force placement of every
assignment, and the count exchange with two gloo ranks.  GPU: R = 2 and 4
virtual ranks on one GPU (every rank's buffers local, the ranks' steps in order
on one stream) give, for every rank's tokens, exactly the bf16 output of the
single-GPU block (moe_forward with all experts): index work and the same per-row
arithmetic, so the comparison is bit-exact."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sigmoid_routed_mixture_b200 import ep

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


# ---------------------------------------------------------------- host side (no GPU)

def test_partition_covers_every_expert_once():
    for E, R in [(256, 8), (16, 3), (64, 4), (5, 5), (7, 1)]:
        f = ep.partition(E, R)
        assert f[0] == 0 and f[-1] == E and len(f) == R + 1
        sizes = np.diff(f)
        assert sizes.min() >= 1 and sizes.max() - sizes.min() <= 1
        assert [ep.owner_of(f, e) for e in range(E)] == sorted(ep.owner_of(f, e) for e in range(E))
    with pytest.raises(ValueError):
        ep.partition(4, 5)
    with pytest.raises(ValueError):
        ep.partition(64, 9)


def brute_force_placement(assign, first):
    """assign[s]: list of (expert, token, slot) of source s in expert-sorted,
    then token order.  Places rows owner by owner: experts ascending, then
    sources ascending, then the source's order.  Returns {(s, t, slot): (owner, row)}."""
    R = len(first) - 1
    place = {}
    for o in range(R):
        row = 0
        for e in range(first[o], first[o + 1]):
            for s in range(R):
                for (ee, t, k) in assign[s]:
                    if ee == e:
                        place[(s, t, k)] = (o, row)
                        row += 1
    return place


@pytest.mark.parametrize("R,E,K", [(2, 8, 2), (3, 16, 4), (4, 16, 4), (8, 8, 8)])
def test_host_plan_matches_brute_force_placement(R, E, K):
    rng = np.random.default_rng(R * 100 + E)
    first = ep.partition(E, R)
    assign, counts = [], np.zeros((R, E), dtype=np.int64)
    for s in range(R):
        T = int(rng.integers(0, 40))
        idx = np.array([rng.permutation(E)[:K] for _ in range(T)]).reshape(T, K)
        a = sorted(((int(idx[t, k]), t, k) for t in range(T) for k in range(K)), key=lambda v: (v[0], v[1]))
        assign.append(a)
        for (e, _, _) in a:
            counts[s, e] += 1
    place = brute_force_placement(assign, first)
    for s in range(R):
        dst_row, _, _ = ep.plan_host(counts, first, s)
        seen = {}
        for (e, t, k) in assign[s]:
            r = seen.get(e, 0)
            seen[e] = r + 1
            assert place[(s, t, k)] == (ep.owner_of(first, e), dst_row[e] + r)
    for o in range(R):
        _, offs, total = ep.plan_host(counts, first, o)
        assert total == counts[:, first[o]:first[o + 1]].sum()
        assert list(np.diff(offs[: first[o + 1] - first[o] + 1])) == list(counts[:, first[o]:first[o + 1]].sum(0))
        assert offs[-1] == offs[-2] == total
        assert sorted(row for (oo, row) in place.values() if oo == o) == list(range(total))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    from sigmoid_routed_mixture_b200 import ep as EP

    E = 16
    rng = np.random.default_rng(7 + rank)
    counts = torch.from_numpy(rng.integers(0, 50, size=E).astype(np.int32))
    allc = EP.exchange_counts(counts)
    first = EP.partition(E, world)
    dst_row, offs, total = EP.plan_host(allc.numpy(), first, rank)
    out[rank] = (allc.numpy().tolist(), dst_row.tolist(), offs.tolist(), total, counts.numpy().tolist())
    dist.destroy_process_group()


def test_count_exchange_and_plan_with_two_gloo_ranks():
    """Every rank ends with the same [R][E] counts (rank s's row is its own),
    the rows rank s sends to each owner start where the rows of the ranks
    before it end, and the two owners receive every assignment once."""
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, free_port(), out), nprocs=world, join=True)
    c0, d0, o0, t0, own0 = out[0]
    c1, d1, o1, t1, own1 = out[1]
    assert c0 == c1 and c0[0] == own0 and c0[1] == own1
    counts = np.array(c0)
    first = ep.partition(16, 2)
    for e in range(16):
        assert d1[e] == d0[e] + counts[0, e]  # rank 1's rows follow rank 0's in every expert
    assert t0 + t1 == counts.sum()
    assert t0 == counts[:, :first[1]].sum() and t1 == counts[:, first[1]:].sum()


# ---------------------------------------------------------------- GPU: virtual ranks

def _virtual_setup(R, T_list, w, seed):
    from sigmoid_routed_mixture_b200 import moe
    from sigmoid_routed_mixture_b200 import workloads as W

    cfg0 = moe.Config.of(w)
    wts = W.expert_weights(w, "cuda")
    _, w_r, b = W.router_inputs(w)
    w_r, b = torch.from_numpy(w_r).cuda(), torch.from_numpy(b).cuda()
    first = ep.partition(w.E, R)
    max_rows = sum(T_list) * w.K
    ranks, xs, refs = [], [], []
    for s, T in enumerate(T_list):
        g = torch.Generator(device="cuda")
        g.manual_seed(seed + s)
        x = torch.randn((T, w.H), generator=g, device="cuda").to(torch.bfloat16)
        cfg = cfg0.replace(T=T)
        ranks.append(ep.EpRank(cfg, first, s, w_r, b, wts["w1"], wts["w3"], wts["w2"], wts["ws1"],
                               wts["ws3"], wts["ws2"], max_rows))
        xs.append(x)
        blk = moe.MoeBlock(cfg, w_r, b, wts["w1"], wts["w3"], wts["w2"], wts["ws1"], wts["ws3"], wts["ws2"])
        refs.append((blk(x).clone(), blk.idx.clone(), blk.counts.clone()))
    return ranks, xs, refs, first


@pytest.mark.gpu
@pytest.mark.parametrize("R,T_list,K,E", [
    (2, [300, 173], 4, 16),        # single-CTA tiles
    (4, [64, 1, 257, 130], 4, 16), # a one-token rank, ragged sizes
    (2, [4096, 4000], 4, 16),      # CTA-pair tiles on both sides
    (4, [512, 0, 300, 2], 8, 32),  # a rank with no tokens
])
def test_virtual_ranks_match_single_gpu_bit_exact(R, T_list, K, E):
    from sigmoid_routed_mixture_b200 import moe
    from sigmoid_routed_mixture_b200 import workloads as W

    w = W.WORKLOADS["tiny"].replace(E=E, K=K, seed=3100 + R)
    ranks, xs, refs, first = _virtual_setup(R, T_list, w, 77)
    for step in range(2):  # the second step reuses every buffer
        ys = ep.virtual_forward(ranks, xs)
        torch.cuda.synchronize()
        for r, y, (y_ref, idx_ref, counts_ref) in zip(ranks, ys, refs):
            assert moe.device_error(r.ws) == 0 and moe.device_error(r.owner_ws) == 0
            assert torch.equal(r.idx, idx_ref)
            assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), "rank %d step %d" % (r.rank, step)
    # the device plan equals the host plan
    counts_all = np.stack([c[: w.E].cpu().numpy() for (_, _, c) in refs])
    for r in ranks:
        dst_row, offs, total = ep.plan_host(counts_all, first, r.rank)
        assert r.dst_row.cpu().numpy().tolist() == dst_row.tolist()
        assert r.recv_offsets.cpu().numpy().tolist() == offs.tolist()
        assert r.recv_sorted[:total].cpu().numpy().tolist() == list(range(total))


@pytest.mark.gpu
def test_small_receive_buffer_is_flagged_not_overrun():
    """A capacity below the rows an owner must take: the rows past it are
    skipped and MOE_ERR_WORKSPACE is flagged; a bad source row id in the return
    is skipped and flagged MOE_ERR_BAD_INDEX."""
    from sigmoid_routed_mixture_b200 import moe
    from sigmoid_routed_mixture_b200 import workloads as W

    w = W.WORKLOADS["tiny"].replace(seed=3200)
    ranks, xs, refs, first = _virtual_setup(2, [200, 100], w, 5)
    for r, x in zip(ranks, xs):
        r.route_and_permute(x)
    counts_all = torch.stack([r.counts[: w.E] for r in ranks])
    for r in ranks:
        ep.plan(r.cfg, first, r.rank, counts_all, r.dst_row, r.recv_offsets, r.recv_sorted, r.ws)
    rows = [int(counts_all[:, first[o]:first[o + 1]].sum()) for o in range(2)]
    ptrs = [[ranks[o].recv_x_ptr(rows[o]) for o in range(2)], [ranks[o].recv_gate.data_ptr() for o in range(2)],
            [ranks[o].recv_src.data_ptr() for o in range(2)]]
    r = ranks[0]
    ep.dispatch(r.cfg, first, 0, r.dst_row, xs[0], r.gate, r.offsets, r.sorted, *ptrs,
                [rows[0] // 2, rows[1] // 2], r.ws)
    torch.cuda.synchronize()
    assert moe.device_error(r.ws) == 4  # MOE_ERR_WORKSPACE
    o = ranks[1]
    o.recv_src[:rows[1]] = torch.tensor([0, 10 ** 6], dtype=torch.int32, device="cuda")
    ep.ret(o.owner_cfg(rows[1]), 2, o.recv_src, [r.slot_outputs_ptr() for r in ranks],
           [rr.cfg.T * rr.cfg.K for rr in ranks], o.owner_ws)
    torch.cuda.synchronize()
    assert moe.device_error(o.owner_ws) == 5  # MOE_ERR_BAD_INDEX
