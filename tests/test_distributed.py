"""The distributed variant (one process per GPU, signs exchanged by a 1-bit
all-gather or an int8 SUM all-reduce).

CPU: the exchange layout and the collectives on two gloo ranks — every slot
the vote reads holds the right rank's signs for the right (matrix, worker).
GPU: two ranks emulated in one process (the exchange done by concatenation /
addition on the device, no collective) give bit for bit the weights of the
single-process step over all their workers, and -- fed every rank's own
signs -- the oracle's majority vote and update give bit for bit the same
weights (the vote matrix, for the local polar step); one NCCL rank runs the
pipelined step() and matches both too."""
import os
import socket

import numpy as np
import pytest
import torch

from sign_muon_optimizer_momentum_b200 import _lib as L
from sign_muon_optimizer_momentum_b200 import distributed as D
from sign_muon_optimizer_momentum_b200 import synthetic as syn

SHAPES = [(64, 96), (96, 64), (33, 147), (256, 256), (5, 40), (128, 640)]


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not os.path.exists(L.LIB_PATH):
        from sign_muon_optimizer_momentum_b200 import build
        build.build()


@pytest.mark.parametrize("variant", ["pack1", "int8"])
@pytest.mark.parametrize("n_groups", [1, 2, 3, 4, 10])
def test_exchange_layout(variant, n_groups):
    Ml = 3
    lay = D.exchange_layout(SHAPES, Ml, n_groups, variant)
    assert 1 <= len(lay.groups) <= min(n_groups, len(SHAPES))
    assert lay.groups[0][0] == 0 and lay.groups[-1][1] == len(SHAPES)
    for (a, b), (c, d) in zip(lay.groups, lay.groups[1:]):
        assert a < b == c < d
    esz = 4 if variant == "pack1" else 1
    for i, (r, c) in enumerate(SHAPES):
        need = L.signmuon_packed_words((r, c)) if variant == "pack1" else r * c
        g = lay.group_of[i]
        assert lay.groups[g][0] <= i < lay.groups[g][1]
        for m in range(Ml):
            off = lay.offsets[i * Ml + m]
            assert (off * esz) % 16 == 0
            nxt = [lay.offsets[u] for u in range(len(lay.offsets))
                   if lay.group_of[u // Ml] == g and lay.offsets[u] > off]
            end = min(nxt) if nxt else lay.group_len[g]
            assert end - off >= need                      # the unit's block holds its signs
    assert (np.array(lay.group_len) * esz % 16 == 0).all()


def test_vote_sign_offsets_order():
    lay = D.exchange_layout(SHAPES, 2, 2, "pack1")
    offs = D.vote_sign_offsets(lay, 3)
    assert len(offs) == len(SHAPES) * 3 * 2
    i, r, m = 4, 2, 1
    g, off = offs[(i * 3 + r) * 2 + m]
    assert g == lay.group_of[i] and off == r * lay.group_len[g] + lay.offsets[i * 2 + m]
    lay8 = D.exchange_layout(SHAPES, 2, 2, "int8")
    assert D.vote_sign_offsets(lay8, 3) == [(lay8.group_of[u // 2], lay8.offsets[u]) for u in range(len(SHAPES) * 2)]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _fill(rank, unit, n, variant):
    """Distinct content per (rank, unit, position)."""
    j = np.arange(n, dtype=np.int64)
    if variant == "pack1":
        return torch.from_numpy(((rank * 1000003 + unit * 7919 + j * 31) & 0x7FFFFFFF).astype(np.int32))
    return torch.from_numpy(np.where((rank + unit + j) % 3 == 0, -1, 1).astype(np.int8))


def _gloo_worker(rank, world, port, variant, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    Ml = 2
    lay = D.exchange_layout(SHAPES, Ml, 3, variant)
    dt = torch.int32 if variant == "pack1" else torch.int8
    local = [torch.zeros(n, dtype=dt) for n in lay.group_len]
    for u, off in enumerate(lay.offsets):
        i = u // Ml
        n = L.signmuon_packed_words(SHAPES[i]) if variant == "pack1" else SHAPES[i][0] * SHAPES[i][1]
        local[lay.group_of[i]][off:off + n] = _fill(rank, u, n, variant)
    gathered = [torch.zeros(world * n, dtype=dt) for n in lay.group_len] if variant == "pack1" else None
    for g in range(len(lay.groups)):
        D.exchange(variant, local[g], gathered[g] if gathered else None)
    ok = True
    src = gathered if variant == "pack1" else local
    offs = D.vote_sign_offsets(lay, world)
    k = 0
    for i, (r_, c_) in enumerate(SHAPES):
        n = L.signmuon_packed_words((r_, c_)) if variant == "pack1" else r_ * c_
        ranks = range(world) if variant == "pack1" else [None]
        for r in ranks:
            for m in range(Ml):
                g, off = offs[k]
                k += 1
                got = src[g][off:off + n]
                if variant == "pack1":
                    want = _fill(r, i * Ml + m, n, variant)
                else:
                    want = sum(_fill(q, i * Ml + m, n, variant).to(torch.int32) for q in range(world)).to(torch.int8)
                ok &= bool(torch.equal(got, want))
    out[rank] = ok
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("variant", ["pack1", "int8"])
def test_gloo_exchange_two_ranks(variant):
    import torch.multiprocessing as mp
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_gloo_worker, args=(world, _free_port(), variant, out), nprocs=world, join=True)
        res = dict(out)
    assert res == {0: True, 1: True}


def _dropout_worker(rank, world, port, out):
    import datetime
    import time
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        out[rank] = "left"                       # drops out before the exchange
        return
    lay = D.exchange_layout(SHAPES, 1, 1, "pack1")
    local = torch.zeros(lay.group_len[0], dtype=torch.int32)
    gathered = torch.zeros(world * lay.group_len[0], dtype=torch.int32)
    t0 = time.time()
    try:
        D.exchange("pack1", local, gathered)
        out[rank] = "no error"
    except Exception as e:                       # the missing rank surfaces as an error
        out[rank] = f"error after {time.time() - t0:.1f}s: {type(e).__name__}"


def test_gloo_exchange_with_a_dropped_rank_raises():
    """A rank that leaves before the exchange makes the collective fail on the
    others within the group's timeout (an exception, not a hang)."""
    import torch.multiprocessing as mp
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_dropout_worker, args=(2, _free_port(), out), nprocs=2, join=True)
        res = dict(out)
    assert res[1] == "left"
    assert res[0].startswith("error after"), res[0]


# ---------------------------------------------------------------------------
# GPU
# ---------------------------------------------------------------------------
def _grads(shapes, M, step, dtype):
    wl = syn.Workload("dist", tuple(shapes), M, 2, "pack1", "f32")
    sig = syn.gradient_signal(wl, seed=5)
    return [syn.worker_gradient(wl, sig[i], i, m, step, seed=5).to(dtype)
            for i in range(len(shapes)) for m in range(M)]


def _unit_signs(buf, off, shape, variant):
    """The {-1,+1} signs of one unit from an exchange buffer (packed words or
    int8 at element offset `off`)."""
    from oracle import signmuon_oracle as O
    r, c = shape
    if variant == "pack1":
        wpr = (c + 31) // 32
        words = buf[off:off + r * wpr].cpu().numpy().view(np.uint32).reshape(r, wpr)
        return O.unpack_signs(words, c)
    return buf[off:off + r * c].cpu().numpy().reshape(r, c)


def _oracle_votes(shapes, layout, local_bufs, variant):
    """The oracle's majority vote of every matrix over all world x local
    workers, from each rank's own (pre-exchange) sign buffers; global worker
    r * local_workers + m."""
    from oracle import signmuon_oracle as O
    Ml = layout.local_workers
    votes = []
    for i, shape in enumerate(shapes):
        g = layout.group_of[i]
        signs = [_unit_signs(bufs[g], layout.offsets[i * Ml + m], shape, variant)
                 for bufs in local_bufs for m in range(Ml)]
        votes.append(O.majority_vote(signs))
    return votes


def _check_against_oracle(shapes, votes, w_prev, w_new, dtype, eta):
    from oracle import signmuon_oracle as O
    wd = "bf16" if dtype == torch.bfloat16 else "f32"
    for i, shape in enumerate(shapes):
        ref = O.apply_update(w_prev[i].double().cpu().numpy(), eta, votes[i], wd)
        assert np.array_equal(w_new[i].double().cpu().numpy(), ref), shape


def _single_process_reference(shapes, M, k, variant, dtype, steps, polar):
    from sign_muon_optimizer_momentum_b200.step import SignMuonStep
    opt = SignMuonStep(shapes, M, k, variant, 0.9, 0.02, dtype, polar=polar)
    w = [syn.gaussian(s, 0.02, "cpu", "Wd", i, dtype=dtype).cuda() for i, s in enumerate(shapes)]
    for t in range(steps):
        opt.step(w, [g.cuda() for g in _grads(shapes, M, t, dtype)])
    torch.cuda.synchronize()
    return [x.cpu() for x in w]


@pytest.mark.gpu
@pytest.mark.parametrize("variant,dtype,polar", [("pack1", torch.bfloat16, False), ("int8", torch.float32, False),
                                                 ("pack1", torch.float32, True)])
def test_two_emulated_ranks_match_single_process(cuda_lib, monkeypatch, variant, dtype, polar):
    monkeypatch.setenv("SIGNMUON_NS_TILE_MODE", "pair")   # same tiles whatever the grouping
    shapes, world, Ml, k, steps = SHAPES, 2, 2, 2, 2
    M = world * Ml
    ref = _single_process_reference(shapes, M, k, variant, dtype, steps, polar)
    ranks = [D.SignMuonDistStep(shapes, Ml, k, variant, 0.9, 0.02, dtype, polar=polar, world_size=world, rank=r,
                                n_groups=3) for r in range(world)]
    ws = [[syn.gaussian(s, 0.02, "cpu", "Wd", i, dtype=dtype).cuda() for i, s in enumerate(shapes)]
          for _ in range(world)]
    for t in range(steps):
        g_all = _grads(shapes, M, t, dtype)              # global worker w = r * Ml + m
        for r, rk in enumerate(ranks):
            mine = [g_all[i * M + r * Ml + m].cuda() for i in range(len(shapes)) for m in range(Ml)]
            rk.local_phase(mine)
        torch.cuda.synchronize()
        # Oracle: the majority vote of every rank's own signs, then the update.
        votes = _oracle_votes(shapes, ranks[0].layout, [[b.clone() for b in rk.local] for rk in ranks], variant)
        w_prev = [[x.clone() for x in w] for w in ws]
        for g in range(len(ranks[0].layout.groups)):     # the exchange, done on the device
            if variant == "pack1":
                cat = torch.cat([rk.local[g] for rk in ranks])
                for rk in ranks:
                    rk.gathered[g].copy_(cat)
            else:
                tot = sum(rk.local[g].to(torch.int32) for rk in ranks).to(torch.int8)
                for rk in ranks:
                    rk.local[g].copy_(tot)
        for rk, w in zip(ranks, ws):
            rk.vote_phase(w)
        torch.cuda.synchronize()
        for rk, w, wp in zip(ranks, ws, w_prev):
            if polar:      # the vote matrix the local polar step starts from
                for i, (r_, c_) in enumerate(shapes):
                    assert np.array_equal(rk.vote[i][:, :c_].double().cpu().numpy(), votes[i])
            else:          # vote + update bit-exact against the oracle
                _check_against_oracle(shapes, votes, wp, w, dtype, 0.02)
    for w in ws:
        for a, b in zip(w, ref):
            assert torch.equal(a.cpu(), b)


@pytest.mark.gpu
@pytest.mark.parametrize("variant,dtype", [("pack1", torch.bfloat16), ("int8", torch.float32)])
def test_nccl_single_rank_step_matches_single_process(cuda_lib, monkeypatch, variant, dtype):
    import datetime
    import torch.distributed as dist
    monkeypatch.setenv("SIGNMUON_NS_TILE_MODE", "pair")
    shapes, Ml, k, steps = SHAPES, 3, 2, 2
    ref = _single_process_reference(shapes, Ml, k, variant, dtype, steps, False)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        opt = D.SignMuonDistStep(shapes, Ml, k, variant, 0.9, 0.02, dtype, n_groups=3)
        w = [syn.gaussian(s, 0.02, "cpu", "Wd", i, dtype=dtype).cuda() for i, s in enumerate(shapes)]
        for t in range(steps):
            w_prev = [x.clone() for x in w]
            opt.step(w, [g.cuda() for g in _grads(shapes, Ml, t, dtype)])
            torch.cuda.synchronize()
            # After the collective (one rank) the local buffers still hold this
            # rank's signs: the oracle's vote + update of them is bit-exact.
            votes = _oracle_votes(shapes, opt.layout, [opt.local], variant)
            _check_against_oracle(shapes, votes, w_prev, w, dtype, 0.02)
        for a, b in zip(w, ref):
            assert torch.equal(a.cpu(), b)
        assert opt.exchange_bytes_per_step() == sum(opt.layout.group_len) * (4 if variant == "pack1" else 1)
    finally:
        dist.destroy_process_group()
