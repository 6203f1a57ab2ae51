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
