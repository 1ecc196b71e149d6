"""Megabatched step (newton_schulz_10_b200/megabatch.py) on several ranks.

CPU, gloo, world sizes 2 and 3: every matrix is split by rows over the
ranks, the momentum shards of each shape travel to the matrix's owner in one
all-to-all, the owner orthogonalises, and one all-to-all brings the update's
rows back. The step's arithmetic is injected: here a stand-in built on the
oracle (momentum, polar approximation, NorMuon, Dion3 selection, update, as
oracle.muon_step computes them), so after the exchange every rank's rows of
W, M and v must equal oracle.muon_step on the whole matrix bit for bit. On
the GPU the same module runs the library's three step parts (see
test_gpu_split_step.py for their equality with muon_step).
"""

import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# several matrices per shape, a shape with fewer rows than ranks, odd row counts
SHAPES = [(12, 20), (12, 20), (12, 20), (7, 9), (7, 9), (20, 6), (2, 8), (12, 20)]


class OracleCompute:
    """The step's arithmetic on CPU tensors, as oracle.muon_step does it."""

    def __init__(self, sp, dion3_frac=None):
        import oracle
        self.O = oracle
        self.sp = sp
        self.frac = dion3_frac

    @property
    def normuon(self):
        return self.sp.normuon

    @property
    def dion3(self):
        return self.frac is not None

    def operand_dtype(self):
        import torch
        return torch.float64

    def scale_dtype(self):
        import torch
        return torch.float64

    def momentum(self, mats):
        import torch
        for (_, M, G, _) in mats:
            if M.shape[0] == 0:
                continue
            Mn, Gn = M.numpy(), G.numpy()
            M.copy_(torch.from_numpy(
                self.O.momentum_accumulate(Mn, Gn) if self.dion3 else self.O.momentum(Mn, Gn, self.sp.mu)))

    def orthogonalize(self, mats, O, scale, sel):
        import torch
        for i, (_, M, _, v) in enumerate(mats):
            Mn = M.numpy()
            rows = Mn.shape[0]
            if self.dion3:
                idx = self.O.select_rows(Mn, self.O.rows_for_fraction(rows, *self.frac), self.sp.select_norm)
            else:
                idx = np.arange(rows)
            Ow = self.O.orthogonalize(Mn[idx, :], self.sp)
            if self.normuon:
                vn = v.numpy()
                v_rows, sc = self.O.normuon(Ow, vn[idx], self.sp.beta2, self.sp.normuon_eps)
                vn[idx] = v_rows.astype(np.float32)
            else:
                sc = np.ones(len(idx))
            o = np.zeros((rows, Mn.shape[1]))
            o[idx] = Ow
            s = np.zeros(rows)
            s[idx] = sc
            O[i].copy_(torch.from_numpy(o))
            scale[i].copy_(torch.from_numpy(s))
            if self.dion3:
                f = np.zeros(rows, np.int32)
                f[idx] = 1
                sel[i].copy_(torch.from_numpy(f))

    def apply_update(self, mats, O, scale, sel):
        import torch
        for i, (W, M, _, _) in enumerate(mats):
            if W.shape[0] == 0:
                continue
            Wn, Mn = W.numpy(), M.numpy()
            rows = np.arange(Wn.shape[0]) if not self.dion3 else np.where(sel[i].numpy() == 1)[0]
            o, s = O[i].numpy(), scale[i].numpy()
            Wn[rows] = (Wn[rows].astype(np.float64) - self.sp.lr * s[rows, None] * o[rows]).astype(np.float32)
            if self.dion3:
                Mn[rows] = (np.float32(self.sp.mu) * Mn[rows]).astype(np.float32)
            W.copy_(torch.from_numpy(Wn))
            M.copy_(torch.from_numpy(Mn))


def _state(j, shape):
    from newton_schulz_10_b200 import inputs
    W = inputs.gaussian(shape, 0.5, 9100 + j, 0)
    M = inputs.gaussian(shape, 0.3, 9100 + j, 2)
    G = inputs.gaussian(shape, 1.0, 9100 + j, 1)
    v = (0.01 + 0.1 * inputs.rng(9100 + j, 3).random(shape[0])).astype(np.float32)
    return W, M, G, v


def _variant(name):
    import oracle
    if name == "muon_normuon":
        return oracle.StepParams(lr=0.1, normuon=True, beta2=0.9, normuon_eps=1e-4), None
    if name == "dion3_normuon":
        return oracle.StepParams(lr=0.1, normuon=True, beta2=0.9, normuon_eps=1e-4, gram=True), (1, 3)
    return oracle.StepParams(lr=0.1), None


def _worker(rank, world, port, variant, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from newton_schulz_10_b200 import megabatch
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sp, frac = _variant(variant)
    shards = []
    for j, shape in enumerate(SHAPES):
        lo, hi = megabatch.row_split(shape[0], world, rank)
        W, M, G, v = _state(j, shape)
        shards.append(tuple(torch.from_numpy(np.ascontiguousarray(a[lo:hi])) for a in (W, M, G, v)))
    step = megabatch.MegabatchedStep(shards, SHAPES, compute=OracleCompute(sp, frac))
    from newton_schulz_10_b200 import inputs
    for it in range(2):
        for j, shape in enumerate(SHAPES):  # a fresh gradient each step
            lo, hi = megabatch.row_split(shape[0], world, rank)
            shards[j][2].copy_(torch.from_numpy(np.ascontiguousarray(
                inputs.gaussian(shape, 1.0, 9300 + j + 17 * it, 1)[lo:hi])))
        step()
    out.put((rank, [tuple(t.numpy().copy() for t in (W, M, v)) for (W, M, _, v) in shards]))
    dist.barrier()
    dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _reference(variant):
    """oracle.muon_step on the whole matrices, the same two steps."""
    import oracle
    from newton_schulz_10_b200 import inputs
    sp, frac = _variant(variant)
    res = []
    for j, shape in enumerate(SHAPES):
        W, M, G, v = _state(j, shape)
        for step in range(2):
            G = inputs.gaussian(shape, 1.0, 9300 + j + 17 * step, 1)
            p = sp if frac is None else oracle.StepParams(**{**sp.__dict__, "k": oracle.rows_for_fraction(
                shape[0], *frac)})
            o = oracle.muon_step(W, M, G, v, p)
            W, M, v = o["W"], o["M"], o["v"]
        res.append((W, M, v))
    return res


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("variant", ["muon", "muon_normuon", "dion3_normuon"])
def test_megabatched_step_equals_single_process(world, variant):
    from newton_schulz_10_b200 import megabatch
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, variant, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    want = _reference(variant)
    for j, shape in enumerate(SHAPES):
        for r in range(world):
            lo, hi = megabatch.row_split(shape[0], world, r)
            for name, a, b in zip("WMv", got[r][j], want[j]):
                assert np.array_equal(a, b[lo:hi]), (variant, world, j, r, name)


def test_owners_balance_each_shape():
    from newton_schulz_10_b200 import megabatch
    own, groups = megabatch.owners(SHAPES, 3)
    for shape, idx in groups.items():
        counts = [sum(1 for j in idx if own[j] == r) for r in range(3)]
        assert max(counts) - min(counts) <= 1
    assert sorted(groups[(12, 20)]) == [0, 1, 2, 7]
    # rows split exactly, in order
    for rows in (2, 7, 12, 20):
        parts = [megabatch.row_split(rows, 3, r) for r in range(3)]
        assert parts[0][0] == 0 and parts[-1][1] == rows
        assert all(parts[r][1] == parts[r + 1][0] for r in range(2))
