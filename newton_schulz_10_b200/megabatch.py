"""Megabatched Muon / Dion3 step over row-sharded matrices on several GPUs.

Section "4. Megabatched Communication" of the Dion3 page: instead of
orthogonalising the matrices in groups of world_size (one communication round
per group), all matrices of one shape form one batch. Every rank packs its
momentum shards of that shape into one all-to-all, each matrix is assembled
on the rank that owns it, every owner orthogonalises all its matrices as one
batched call, and one all-to-all per shape scatters the orthogonalised rows
back. The rounds per step are two per distinct shape, whatever the number of
matrices.

Layout (FSDP-style): matrix j (rows x cols, the same on every rank) is split
by rows; rank r holds rows [lo, hi) of it as given by `row_split`. The
weights, the momentum and the NorMuon second moments stay sharded; only the
momentum (with v for NorMuon) travels to the owner, and only the update (the
orthogonalised rows in the operand type, their row scales, the Dion3
selection and the new v) travels back. The owner of the k-th matrix of a
shape group is rank (offset + k) mod world_size, with the offset running on
across groups, so every rank owns the same number of matrices of each shape
(give or take one) and so the same Newton-Schulz FLOPs.

The arithmetic is the library's: muon_momentum on the local shards,
muon_orthogonalize on the owned full matrices, muon_apply_update on the local
shards. Those three calls in sequence equal muon_step bit for bit, so the
megabatched step gives every rank exactly the rows a single-GPU step would.
The exchange uses torch.distributed (NCCL over NVLink between GPUs); peer
data lands in this GPU's own memory before any kernel reads it. This module
only moves and packs data.
"""

from __future__ import annotations

from dataclasses import dataclass


def row_split(rows: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [lo, hi) of a rows-row matrix held by `rank`: the first
    rows % world ranks hold one row more than the others."""
    base, extra = divmod(rows, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def owners(shapes, world: int):
    """Owner rank of every matrix and the shape groups (shape -> matrix
    indices, in order of first appearance)."""
    groups = {}
    for j, s in enumerate(shapes):
        groups.setdefault(tuple(s), []).append(j)
    own = [0] * len(shapes)
    offset = 0
    for idx in groups.values():
        for k, j in enumerate(idx):
            own[j] = (offset + k) % world
        offset += len(idx)
    return own, groups


class LibmuonCompute:
    """The library's three step parts on CUDA tensors (the product path)."""

    def __init__(self, params):
        from newton_schulz_10_b200 import muon as mu
        self.mu = mu
        self.p = params
        self.ws = None

    def operand_dtype(self):
        return self.mu.operand_dtype(self.p)

    def scale_dtype(self):
        import torch
        return torch.float32

    def momentum(self, mats):
        self.mu.momentum(mats, self.p)

    def orthogonalize(self, mats, O, scale, sel):
        need = self.mu.workspace_size(mats, self.p)
        if self.ws is None or self.ws.numel() < need:
            self.ws = self.mu.workspace(need, mats[0][1].device)
        self.mu.orthogonalize(mats, self.p, O, scale, sel, ws=self.ws)

    def apply_update(self, mats, O, scale, sel):
        self.mu.apply_update(mats, self.p, O, scale, sel)

    @property
    def normuon(self):
        return bool(self.p.normuon)

    @property
    def dion3(self):
        return bool(self.p.dion3)


_ALIGN = 16  # bytes: every packed piece starts on a 16-byte boundary


def _pad(n: int) -> int:
    return (n + _ALIGN - 1) // _ALIGN * _ALIGN


@dataclass
class _Piece:
    offset: int
    nbytes: int


class MegabatchedStep:
    """One optimizer step over row shards, megabatched by shape.

    shards[j] = (W, M, G, v) of matrix j on this rank (rows of the shard x
    cols; v may be None without NorMuon); shapes[j] = full (rows, cols).
    compute: the step parts (LibmuonCompute(params) by default for CUDA
    tensors); group: the torch.distributed process group (default group)."""

    def __init__(self, shards, shapes, params=None, compute=None, group=None):
        import torch
        import torch.distributed as dist

        self.torch = torch
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.shards = list(shards)
        self.shapes = [tuple(s) for s in shapes]
        self.compute = compute if compute is not None else LibmuonCompute(params)
        self.own, self.groups = owners(self.shapes, self.world)
        self.device = self.shards[0][1].device if self.shards else torch.device("cpu")
        for j, (sh, (rows, cols)) in enumerate(zip(self.shards, self.shapes)):
            lo, hi = row_split(rows, self.world, self.rank)
            if tuple(sh[1].shape) != (hi - lo, cols):
                raise ValueError(f"matrix {j}: shard {tuple(sh[1].shape)} is not rows [{lo}, {hi}) x {cols}")

    # -- packing helpers ------------------------------------------------------

    def _bytes(self, t):
        return t.contiguous().view(-1).view(self.torch.uint8)

    def _layout(self, pieces_per_peer):
        """Offsets of the pieces to or from every peer in one uint8 buffer;
        returns (total bytes, bytes per peer, offsets per peer)."""
        per_peer, offsets, total = [], [], 0
        for pieces in pieces_per_peer:
            start = total
            offs = []
            for nb in pieces:
                offs.append(_Piece(total, nb))
                total += _pad(nb)
            per_peer.append(total - start)
            offsets.append(offs)
        return total, per_peer, offsets

    def _exchange(self, send, send_sizes, recv_sizes):
        recv = self.torch.empty(sum(recv_sizes), dtype=self.torch.uint8, device=self.device)
        self.dist.all_to_all_single(recv, send, recv_sizes, send_sizes, group=self.group)
        return recv

    def _view(self, buf, piece, dtype, shape):
        return buf[piece.offset:piece.offset + piece.nbytes].view(dtype).view(shape)

    # -- the step -------------------------------------------------------------

    def __call__(self) -> None:
        torch = self.torch
        c = self.compute
        world, me = self.world, self.rank
        f32, i32 = torch.float32, torch.int32
        op_dt, sc_dt = c.operand_dtype(), c.scale_dtype()
        op_es = torch.empty((), dtype=op_dt).element_size()
        sc_es = torch.empty((), dtype=sc_dt).element_size()

        # 1. momentum on the local shards
        c.momentum([(W, M, G, v) for (W, M, G, v) in self.shards])

        # 2. one all-to-all per shape group: momentum (and v) shards to owners
        full = {}  # j -> (M, v) assembled on its owner
        for (rows, cols), idx in self.groups.items():
            mine = [j for j in idx if self.own[j] == me]
            send_p = [[] for _ in range(world)]
            for j in idx:
                lo, hi = row_split(rows, world, me)
                send_p[self.own[j]] += [(hi - lo) * cols * 4] + ([(hi - lo) * 4] if c.normuon else [])
            recv_p = [[] for _ in range(world)]
            for r in range(world):
                lo, hi = row_split(rows, world, r)
                for j in mine:
                    recv_p[r] += [(hi - lo) * cols * 4] + ([(hi - lo) * 4] if c.normuon else [])
            stot, ssz, soff = self._layout(send_p)
            rtot, rsz, roff = self._layout(recv_p)
            send = torch.zeros(stot, dtype=torch.uint8, device=self.device)
            k = [0] * world
            for j in idx:
                d = self.own[j]
                W, M, G, v = self.shards[j]
                pc = soff[d][k[d]]
                send[pc.offset:pc.offset + pc.nbytes] = self._bytes(M)
                k[d] += 1
                if c.normuon:
                    pc = soff[d][k[d]]
                    send[pc.offset:pc.offset + pc.nbytes] = self._bytes(v)
                    k[d] += 1
            recv = self._exchange(send, ssz, rsz)
            for j in mine:
                full[j] = (torch.empty((rows, cols), dtype=f32, device=self.device),
                           torch.empty(rows, dtype=f32, device=self.device) if c.normuon else None)
            for r in range(world):
                lo, hi = row_split(rows, world, r)
                k = 0
                for j in mine:
                    full[j][0][lo:hi] = self._view(recv, roff[r][k], f32, (hi - lo, cols))
                    k += 1
                    if c.normuon:
                        full[j][1][lo:hi] = self._view(recv, roff[r][k], f32, (hi - lo,))
                        k += 1

        # 3. the owner orthogonalises all its matrices as one batch
        owned = sorted(full)
        O = {j: torch.empty(self.shapes[j], dtype=op_dt, device=self.device) for j in owned}
        scale = {j: torch.empty(self.shapes[j][0], dtype=sc_dt, device=self.device) for j in owned}
        sel = {j: torch.empty(self.shapes[j][0], dtype=i32, device=self.device) for j in owned} if c.dion3 else None
        if owned:
            c.orthogonalize([(None, full[j][0], None, full[j][1]) for j in owned], [O[j] for j in owned],
                            [scale[j] for j in owned], [sel[j] for j in owned] if c.dion3 else None)

        # 4. one all-to-all per shape group: the update's rows back to the shards
        upd = {}  # j -> (O, scale, sel, v) rows of this rank's shard
        for (rows, cols), idx in self.groups.items():
            mine = [j for j in idx if self.own[j] == me]

            def pieces(nrows):
                p = [nrows * cols * op_es, nrows * sc_es]
                if c.dion3:
                    p.append(nrows * 4)
                if c.normuon:
                    p.append(nrows * 4)
                return p

            send_p = [[] for _ in range(world)]
            for r in range(world):
                lo, hi = row_split(rows, world, r)
                for j in mine:
                    send_p[r] += pieces(hi - lo)
            recv_p = [[] for _ in range(world)]
            lo_me, hi_me = row_split(rows, world, me)
            for j in idx:
                recv_p[self.own[j]] += pieces(hi_me - lo_me)
            stot, ssz, soff = self._layout(send_p)
            rtot, rsz, roff = self._layout(recv_p)
            send = torch.zeros(stot, dtype=torch.uint8, device=self.device)
            for r in range(world):
                lo, hi = row_split(rows, world, r)
                k = 0
                for j in mine:
                    parts = [O[j][lo:hi], scale[j][lo:hi]]
                    if c.dion3:
                        parts.append(sel[j][lo:hi])
                    if c.normuon:
                        parts.append(full[j][1][lo:hi])
                    for t in parts:
                        pc = soff[r][k]
                        send[pc.offset:pc.offset + pc.nbytes] = self._bytes(t)
                        k += 1
            recv = self._exchange(send, ssz, rsz)
            k = [0] * world
            n = hi_me - lo_me
            for j in idx:
                src = self.own[j]
                pcs = roff[src]
                o = self._view(recv, pcs[k[src]], op_dt, (n, cols))
                s = self._view(recv, pcs[k[src] + 1], sc_dt, (n,))
                k[src] += 2
                f = None
                if c.dion3:
                    f = self._view(recv, pcs[k[src]], i32, (n,))
                    k[src] += 1
                v = None
                if c.normuon:
                    v = self._view(recv, pcs[k[src]], f32, (n,))
                    k[src] += 1
                upd[j] = (o, s, f, v)

        # 5. the update on the local shards (and the new second moments)
        mats = [(W, M, G, v) for (W, M, G, v) in self.shards]
        c.apply_update(mats, [upd[j][0] for j in range(len(mats))], [upd[j][1] for j in range(len(mats))],
                       [upd[j][2] for j in range(len(mats))] if c.dion3 else None)
        if c.normuon:
            for j, (W, M, G, v) in enumerate(self.shards):
                v.copy_(upd[j][3])
