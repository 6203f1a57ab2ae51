"""Peer-pointer exchange of the expert-parallel forward with gloo ranks on the CPU.

Every rank exports (IPC handle, offset) of its buffer; every other rank's
allocation is mapped once, and a handle seen again (a second buffer of an
allocation already mapped) reuses that mapping.  The CUDA IPC calls are replaced by fakes
(a handle names its rank and allocation; opening returns a made-up base), so no
device is needed; the C entry points themselves are checked in test_abi.py.
"""
import os
import socket

import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


FAKE_BASE = {0: 0x7000_0000_0000, 1: 0x7100_0000_0000, 2: 0x7200_0000_0000}


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from mixture_experts_layer_persistent_b200.ep import exchange_pointers

    opened = []

    # rank r's buffers live in allocation "A<r>": x at offset 256, state at offset 4096
    def export(ptr):
        return (f"A{rank}".encode().ljust(64, b"\0"), ptr - 0x1000_0000 * (rank + 1))

    def open_(handle, offset):
        assert offset == 0
        opened.append(handle)
        r = int(handle.rstrip(b"\0")[1:])
        return FAKE_BASE[r]

    local = 0x1000_0000 * (rank + 1)
    xs, ox = exchange_pointers(local + 256, export=export, open_=open_)
    ss, os_ = exchange_pointers(local + 4096, export=export, open_=open_, opened=ox)
    q.put((rank, xs, ss, sorted(ox.values()), sorted(os_.values()), len(opened)))
    dist.barrier()
    dist.destroy_process_group()


def test_three_ranks_map_each_peer_allocation_once():
    world = 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, xs, ss, ox, os_, n_open in res:
        assert len(xs) == len(ss) == world
        for r in range(world):
            if r == rank:           # own buffers: the local pointers, never opened
                assert xs[r] == 0x1000_0000 * (rank + 1) + 256 and ss[r] == 0x1000_0000 * (rank + 1) + 4096
            else:                   # peers: mapped base + the exported offset
                assert xs[r] == FAKE_BASE[r] + 256 and ss[r] == FAKE_BASE[r] + 4096
        peers = sorted(FAKE_BASE[r] for r in range(world) if r != rank)
        assert ox == peers and os_ == peers
        assert n_open == world - 1     # x and state share each peer's allocation: mapped once


def _rank_worker(rank, world, port, q):
    """EPRank's phase order on two gloo ranks, with the C entry points, the IPC calls
    and the CUDA stream calls replaced by recorders (CPU tensors stand in for device
    buffers)."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import torch
    from mixture_experts_layer_persistent_b200 import abi, ep, make_cfg

    calls = []
    torch.cuda.synchronize = lambda *a, **k: None

    class _S:
        cuda_stream = 0
    torch.cuda.current_stream = lambda *a, **k: _S()
    abi.moe_ep_ipc_handle = lambda ptr: (f"R{rank}".encode().ljust(64, b"\0"), 0)
    abi.moe_ep_ipc_open = lambda h, off: 0x7000_0000 + int(h.rstrip(b"\0")[1:]) * 0x100_0000
    abi.moe_ep_ipc_close = lambda p, off: calls.append(("close", p))
    for name in ("moe_ep_route", "moe_ep_experts", "moe_ep_combine", "moe_ep_bwd_experts", "moe_ep_bwd_combine"):
        setattr(abi, name, (lambda n: (lambda *a: calls.append((n, a))))(name))
    real_all_reduce = dist.all_reduce

    def all_reduce(t, *a, **k):
        calls.append(("barrier",))
        return real_all_reduce(t, *a, **k)
    dist.all_reduce = all_reduce

    cfg = make_cfg(16, 256, 8, 128, 2)
    r = ep.EPRank(cfg, {"router_w": torch.zeros(8, 256), "w_gate_up": torch.zeros(4, 256, 256),
                        "w_down": torch.zeros(4, 256, 128)}, training=True, device="cpu")
    r.forward(y=torch.empty(16, 256, dtype=torch.bfloat16))
    r.backward({"dx": torch.empty(16, 256, dtype=torch.bfloat16), "dw_gate_up": torch.empty(4, 256, 256),
                "dw_down": torch.empty(4, 256, 128), "drouter_w": torch.empty(8, 256)})
    r.close()
    order = [c[0] for c in calls]
    ex = [c for c in calls if c[0] == "moe_ep_experts"][0][1]
    bx = [c for c in calls if c[0] == "moe_ep_bwd_experts"][0][1]
    q.put((rank, order, list(ex[4]), list(ex[5]), list(bx[3]), list(bx[4]), r.x.data_ptr(), r.state.data_ptr(),
           r.dy.data_ptr(), r.bwd.data_ptr()))
    dist.barrier()
    dist.destroy_process_group()


def test_rank_phases_are_separated_by_barriers():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, order, xs, ss, dys, bws, x, st, dy, bw in res:
        assert order == ["moe_ep_route", "barrier", "moe_ep_experts", "barrier", "moe_ep_combine",
                         "barrier", "moe_ep_bwd_experts", "barrier", "moe_ep_bwd_combine", "close"], order
        other = 1 - rank
        peer = 0x7000_0000 + other * 0x100_0000
        # pointer tables by rank: own buffers as they are, the peer's through its one mapping
        for table, own in ((xs, x), (ss, st), (dys, dy), (bws, bw)):
            assert table[rank] == own and table[other] == peer, (rank, table)
