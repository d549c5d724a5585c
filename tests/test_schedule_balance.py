"""Work balance of the forward's persistent hand-out (CPU, no GPU).

The tile order and the snake hand-out are restated in ``protocol_model``
(``decode``, ``Sim.tiles``), the same way the kernel computes them.  Work per
CTA is counted in key blocks processed by its Q tiles (tile-blocks), the unit
the kernel's time per work tile is proportional to apart from a fixed cost
per work tile.  The figures below are the design's balance, stated in the
design notes; the test keeps them from drifting."""
import pytest

import protocol_model as pm

SMS = 148


def imbalance(N, B, H, causal, QS=2):
    p = pm.P(N=N, causal=causal, QS=QS, KVS=4, B=B, H=H)
    G = min(SMS, p.num_tiles)
    work = []
    for c in range(G):
        sim = pm.Sim(p, G, c, 0)
        w = 0
        for t in sim.tiles():
            ti = pm.decode(p, t)
            w += sum(ti['hi'][s] - ti['lo'][s] for s in range(QS))
        work.append(w)
    total = sum(work)
    # every tile-block of the problem is handed out exactly once
    nq = (N + 127) // 128
    expect = B * H * (nq * (nq + 1) // 2 if causal else nq * nq)
    assert total == expect
    return max(work) * G / total


@pytest.mark.parametrize("N,B,H,causal,QS,bound", [
    (4096, 4, 16, False, 2, 1.02),    # non-causal: equal tiles
    (2048, 1, 128, True, 2, 1.04),    # causal H=128 N=2048
    (4096, 4, 16, True, 2, 1.03),
    (8192, 2, 16, True, 2, 1.02),
    (16384, 1, 16, True, 2, 1.02),
    (512, 32, 16, True, 2, 1.08),
    (1024, 16, 16, True, 2, 1.12),    # the worst: 4 tile lengths over 6.9 rounds
    (8192, 1, 8, True, 1, 1.07),      # d = 256: one Q tile per work tile
])
def test_longest_first_snake_balances_the_work(N, B, H, causal, QS, bound):
    assert imbalance(N, B, H, causal, QS) <= bound


def bwd_imbalance(B, H, N, causal, kv):
    """The backward kernels' persistent hand-out, restated: units in (b, h)
    order (non-causal) or longest first (causal: key block 0 of every head for
    dK/dV, the last query block for dQ), snake over min(units, SMs) CTAs;
    work = streamed blocks per unit."""
    nblk = (N + 127) // 128
    units = B * H * nblk
    G = min(SMS, units)

    def blocks(u):
        if causal:
            rank = u // (B * H)
            blk = rank if kv else nblk - 1 - rank
        else:
            blk = u % nblk
        first = blk if (kv and causal) else 0
        last = blk if (not kv and causal) else nblk - 1
        return last - first + 1

    work = [0] * G
    r = 0
    while r * G < units:
        for c in range(G):
            u = r * G + ((G - 1 - c) if r & 1 else c)
            if u < units:
                work[c] += blocks(u)
        r += 1
    assert sum(work) == B * H * (nblk * (nblk + 1) // 2 if causal else nblk * nblk)
    return max(work) * G / sum(work)


@pytest.mark.parametrize("B,H,N,causal", [(4, 16, 4096, False), (4, 16, 4096, True),
                                           (16, 16, 1024, False), (16, 16, 1024, True),
                                           (1, 16, 16384, True)])
@pytest.mark.parametrize("kv", [True, False])
def test_backward_hand_out_balances_the_work(B, H, N, causal, kv):
    assert bwd_imbalance(B, H, N, causal, kv) <= 1.015
