"""The forward kernel's mbarrier protocol, run in a CPU model
(``tests/protocol_model.py``) over schedules that cover every kernel
configuration: the ring depths (2, 4, 5 and 10 slots), one and two Q
tiles per work tile, causal and non-causal, a local window, packed
variable-length sequences with empty and partial tiles, and CTAs with one or
several work tiles.  Random completion times, several seeds each.

Each run must finish without deadlock, without a wait that a parity test
could misread (barrier not exactly one phase short), without O being
overwritten before the epilogue read it, without a ring slot being reloaded
before its staged O was stored, and with every P V product reading the P
half written for it, never overwritten while it reads."""
import pytest

import protocol_model as pm

CASES = [
    dict(N=2048, causal=False, QS=2, KVS=4, B=4, H=16),
    dict(N=2048, causal=True, QS=2, KVS=4, B=4, H=16),
    dict(N=8192, causal=True, QS=1, KVS=2, B=1, H=8),
    dict(N=8192, causal=True, QS=1, KVS=2, B=1, H=8, o_tma=False),
    dict(N=777, causal=True, QS=2, KVS=10, B=2, H=3),
    dict(N=1024, causal=True, QS=2, KVS=4, B=2, H=2, left=100),
    dict(N=600, causal=True, QS=2, KVS=4, lens=[1, 7, 128, 0, 129, 300, 513, 256], H=3),
    dict(N=1000, causal=False, QS=2, KVS=10, B=1, H=2, left=64, right=3),
    # e4m3: d = 128 with a 10-slot ring, d = 256 with 5 slots; O by direct stores
    dict(N=2048, causal=False, QS=2, KVS=10, B=2, H=4, o_tma=False),
    dict(N=4096, causal=True, QS=1, KVS=5, B=1, H=4, o_tma=False),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(f"{k}{v}" for k, v in c.items()
                                                               if k != "lens"))
def test_protocol_runs_clean(case):
    p = pm.P(**case)
    G = min(p.num_tiles, 148)
    for cta in sorted({0, G // 2, G - 1}):
        for seed in range(2):
            sim = pm.Sim(p, G, cta, seed)
            r = sim.run()
            assert r == "ok", (cta, seed, r)
            assert not sim.aliased, (cta, seed, sim.aliased[:3])
            assert not sim.hazards, (cta, seed, sim.hazards[:3])


def test_model_flags_a_shared_full_barrier():
    """The model is not vacuous: with one full barrier per slot shared by the
    K, V and O uses (the first design of the ring), the 2-slot ring shows
    waits issued two phases away, which a parity test misreads."""
    p = pm.P(N=8192, causal=True, QS=1, KVS=2, B=1, H=8)
    bad = 0
    for cta in (0, 74, 147):
        for seed in range(2):
            sim = pm.Sim(p, 148, cta, seed, shared_full=True)
            r = sim.run(max_steps=400000)
            bad += (r != "ok") or bool(sim.aliased) or bool(sim.hazards)
    assert bad > 0


def test_model_flags_a_p_half_written_before_its_hand_over():
    """The model checks the shared P buffer's data too: softmax groups that
    write their half without waiting for the previous user's P V K-steps to
    end overwrite P that a product still reads, in some schedule."""
    p = pm.P(N=2048, causal=False, QS=2, KVS=4, B=1, H=2)
    bad = 0
    for cta in (0, 1):
        for seed in range(3):
            sim = pm.Sim(p, 2, cta, seed, skip_pfree=True)
            r = sim.run(max_steps=400000)
            bad += (r != "ok") or bool(sim.hazards)
    assert bad > 0


def test_model_flags_an_s_buffer_overwritten_before_it_was_read():
    """Likewise for the S buffers: an S thread that issues S(j+1) of a Q tile
    without waiting for its softmax to have read S(j) hands the softmax the
    wrong block's scores in some schedule."""
    p = pm.P(N=2048, causal=False, QS=2, KVS=4, B=1, H=2)
    bad = 0
    for cta in (0, 1):
        for seed in range(3):
            sim = pm.Sim(p, 2, cta, seed, skip_sfree=True)
            r = sim.run(max_steps=400000)
            bad += (r != "ok") or bool(sim.hazards)
    assert bad > 0


def test_model_flags_a_q_buffer_reloaded_too_early():
    """And for the Q buffer: loading the next work tile's Q without waiting
    for this tile's last S product shows an S reading the wrong Q in some
    schedule."""
    # a deep ring (d = 64) lets the producer run a work tile ahead
    p = pm.P(N=512, causal=False, QS=2, KVS=10, B=2, H=8)
    bad = 0
    for cta in (0, 1):
        for seed in range(3):
            sim = pm.Sim(p, 2, cta, seed, skip_qempty=True)
            r = sim.run(max_steps=400000)
            bad += (r != "ok") or bool(sim.hazards)
    assert bad > 0
