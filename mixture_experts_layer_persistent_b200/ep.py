"""Expert parallelism around the C ABI (forward and backward): buffers, peer
pointers and the order of the phases.  All arithmetic runs in libmok's kernels (moe_ep_* in
include/mok.h).

"Cursor åpner megakernelen…" (the pull-versus-push paragraph): the rank that
owns an expert pulls the token rows routed to it and pushes each output row
back to its token's rank.  Rank r owns the routed experts
[r E/world, (r+1) E/world); cfg.T is the tokens of one rank.

Two ways to place the ranks:

* ``EPWorld`` -- every rank on the current device, one buffer set per rank,
  the phases in stream order (route on every rank, then every rank's experts,
  then every rank's combine).
* ``EPRank`` -- one process per GPU under torch.distributed.  The ranks'
  x and state buffers are mapped into every process through CUDA IPC handles
  (``exchange_pointers``), and a one-element all-reduce on the stream
  separates the phases: it ends on a rank only after every rank's earlier
  kernels, so no kernel waits on another GPU.
"""
from __future__ import annotations

import torch

from . import abi
from .layer import make_params


def split_params(params: dict, world: int, rank: int, E: int) -> dict:
    """Rank `rank`'s share of a full layer's parameters: its experts' slices of
    w_gate_up / w_down (views), everything else shared."""
    if E % world:
        raise ValueError("E must be a multiple of world")
    el = E // world
    out = dict(params)
    for n in ("w_gate_up", "w_down"):
        out[n] = params[n][rank * el:(rank + 1) * el]
    return out


def _grads(g: dict):
    return abi.moe_grads(*(None if g.get(n) is None else g[n].data_ptr() for n in
                           ("dx", "dw_gate_up", "dw_down", "drouter_w", "dws_gate_up", "dws_down")))


def new_rank_grads(cfg: abi.moe_cfg, world: int, device) -> dict:
    """Gradient tensors of one rank: dx and the router / shared-expert gradients of
    its tokens, dw_* of its own experts."""
    c, el = cfg, cfg.E // world
    g = {"dx": torch.empty((c.T, c.H), dtype=torch.bfloat16, device=device),
         "dw_gate_up": torch.empty((el, 2 * c.I, c.H), dtype=torch.bfloat16, device=device),
         "dw_down": torch.empty((el, c.H, c.I), dtype=torch.bfloat16, device=device),
         "drouter_w": torch.empty((c.E, c.H), dtype=torch.float32, device=device),
         "dws_gate_up": None, "dws_down": None}
    if c.n_shared:
        g["dws_gate_up"] = torch.empty((c.n_shared, 2 * c.I, c.H), dtype=torch.bfloat16, device=device)
        g["dws_down"] = torch.empty((c.n_shared, c.H, c.I), dtype=torch.bfloat16, device=device)
    return g


class EPWorld:
    """All `world` ranks of an expert-parallel layer on the current device."""

    def __init__(self, cfg: abi.moe_cfg, world: int, rank_params: list, training: bool = False, device=None):
        if len(rank_params) != world:
            raise ValueError("one parameter dict per rank")
        self.cfg, self.world, self.training = cfg, world, training
        self.device = torch.device(device or "cuda")
        self.state_bytes, self.scratch_bytes, self.bwd_bytes = abi.moe_ep_size(cfg, world, training)
        mk = lambda n: torch.empty(n, dtype=torch.uint8, device=self.device)
        self.states = [mk(self.state_bytes) for _ in range(world)]
        self.scratch = [mk(self.scratch_bytes) for _ in range(world)]
        self.bwd = [mk(self.bwd_bytes) for _ in range(world)] if training else None
        self.params = rank_params            # keeps the tensors alive
        self.cparams = [make_params(p) for p in rank_params]
        self.xs = None

    def forward(self, xs: list, ys: list = None) -> list:
        c, W = self.cfg, self.world
        if len(xs) != W:
            raise ValueError("one x per rank")
        if ys is None:
            ys = [torch.empty((c.T, c.H), dtype=torch.bfloat16, device=self.device) for _ in range(W)]
        st = torch.cuda.current_stream(self.device).cuda_stream
        xp = [x.data_ptr() for x in xs]
        sp = [s.data_ptr() for s in self.states]
        for r in range(W):
            abi.moe_ep_route(c, W, r, xp[r], self.cparams[r], sp[r], self.state_bytes, st)
        for r in range(W):
            abi.moe_ep_experts(c, W, r, self.training, xp, sp, self.cparams[r], self.scratch[r].data_ptr(),
                               self.scratch_bytes, st)
        for r in range(W):
            abi.moe_ep_combine(c, W, r, sp[r], ys[r].data_ptr(), st)
        self.xs = xs
        return ys

    def backward(self, dys: list, grads: list = None) -> list:
        """Per-rank gradients after a training forward of the same xs (new_rank_grads)."""
        c, W = self.cfg, self.world
        if not self.training or self.xs is None:
            raise RuntimeError("backward needs a training forward first")
        if grads is None:
            grads = [new_rank_grads(c, W, self.device) for _ in range(W)]
        st = torch.cuda.current_stream(self.device).cuda_stream
        dp = [d.data_ptr() for d in dys]
        bp = [b.data_ptr() for b in self.bwd]
        cg = [_grads(g) for g in grads]
        for r in range(W):
            abi.moe_ep_bwd_experts(c, W, r, dp, bp, self.cparams[r], cg[r], self.scratch[r].data_ptr(),
                                   self.scratch_bytes, st)
        for r in range(W):
            abi.moe_ep_bwd_combine(c, W, r, self.xs[r].data_ptr(), self.cparams[r], self.states[r].data_ptr(),
                                   bp[r], self.bwd_bytes, cg[r], st)
        return grads


def exchange_pointers(local_ptr: int, group=None, export=None, open_=None, opened=None):
    """Every rank's pointer to the same buffer role, as this process addresses it.

    Each rank exports (IPC handle, offset) of local_ptr's allocation; every
    other rank's allocation is opened once: pass the `opened` dict of earlier
    calls so that a buffer in an allocation already mapped reuses that mapping
    (CUDA maps one allocation once per process).  Returns (pointers by rank,
    {handle: mapped base}, to close later).
    """
    import torch.distributed as dist
    export = export or abi.moe_ep_ipc_handle
    open_ = open_ or abi.moe_ep_ipc_open
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    mine = export(local_ptr)
    allh = [None] * world
    dist.all_gather_object(allh, mine, group=group)
    ptrs = []
    opened = {} if opened is None else opened
    for r, (h, off) in enumerate(allh):
        if r == rank:
            ptrs.append(int(local_ptr))
            continue
        base = opened.get(h)
        if base is None:
            base = open_(h, 0)
            opened[h] = base
        ptrs.append(base + off)
    return ptrs, opened


class EPRank:
    """This process's rank of an expert-parallel layer (one GPU per process).

    x goes into ``self.x`` and dy into ``self.dy`` (peers read both);
    ``forward`` runs route, barrier, experts, barrier, combine on the current
    stream, ``backward`` barrier, experts, barrier, combine.
    """

    def __init__(self, cfg: abi.moe_cfg, params: dict, training: bool = False, group=None, device=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.cfg = cfg
        self.training = training
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.device = torch.device(device or "cuda")
        self.state_bytes, self.scratch_bytes, self.bwd_bytes = abi.moe_ep_size(cfg, self.world, training)
        mk = lambda n: torch.empty(n, dtype=torch.uint8, device=self.device)
        self.state = mk(self.state_bytes)
        self.scratch = mk(self.scratch_bytes)
        self.bwd = mk(self.bwd_bytes) if training else None
        self.x = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=self.device)
        self.dy = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=self.device) if training else None
        self.params = params
        self.cparams = make_params(params)
        self._flag = torch.zeros(1, dtype=torch.int32, device=self.device)
        torch.cuda.synchronize(self.device)          # buffers exist before peers map them
        self.x_ptrs, self._opened = exchange_pointers(self.x.data_ptr(), group)
        self.state_ptrs, self._opened = exchange_pointers(self.state.data_ptr(), group, opened=self._opened)
        if training:
            self.dy_ptrs, self._opened = exchange_pointers(self.dy.data_ptr(), group, opened=self._opened)
            self.bwd_ptrs, self._opened = exchange_pointers(self.bwd.data_ptr(), group, opened=self._opened)

    def _barrier(self):
        self.dist.all_reduce(self._flag, group=self.group)

    def forward(self, y: torch.Tensor = None) -> torch.Tensor:
        c, W, r = self.cfg, self.world, self.rank
        if y is None:
            y = torch.empty((c.T, c.H), dtype=torch.bfloat16, device=self.device)
        st = torch.cuda.current_stream(self.device).cuda_stream
        abi.moe_ep_route(c, W, r, self.x.data_ptr(), self.cparams, self.state.data_ptr(), self.state_bytes, st)
        self._barrier()
        abi.moe_ep_experts(c, W, r, self.training, self.x_ptrs, self.state_ptrs, self.cparams,
                           self.scratch.data_ptr(), self.scratch_bytes, st)
        self._barrier()
        abi.moe_ep_combine(c, W, r, self.state.data_ptr(), y.data_ptr(), st)
        return y

    def backward(self, grads: dict = None) -> dict:
        c, W, r = self.cfg, self.world, self.rank
        grads = grads or new_rank_grads(c, W, self.device)
        cg = _grads(grads)
        st = torch.cuda.current_stream(self.device).cuda_stream
        self._barrier()                              # every rank's dy is in place
        abi.moe_ep_bwd_experts(c, W, r, self.dy_ptrs, self.bwd_ptrs, self.cparams, cg, self.scratch.data_ptr(),
                               self.scratch_bytes, st)
        self._barrier()
        abi.moe_ep_bwd_combine(c, W, r, self.x.data_ptr(), self.cparams, self.state.data_ptr(),
                               self.bwd.data_ptr(), self.bwd_bytes, cg, st)
        return grads

    def close(self):
        torch.cuda.synchronize(self.device)
        for base in self._opened.values():
            abi.moe_ep_ipc_close(base, 0)
        self._opened = {}
