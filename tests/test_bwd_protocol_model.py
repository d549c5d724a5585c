"""The backward kernels' mbarrier protocol, run in a CPU model
(``tests/bwd_protocol_model.py``) for the three kernel shapes: the dK/dV
kernel with one dP region (d = 128), the dK/dV kernel with two (d = 64) and
the dQ kernel (two), over 1 to 32 streamed blocks, random completion times,
several seeds each.

Each run must finish without deadlock, without a wait that a parity test
could misread, and with every MMA and compute warp reading the operand of
its own step (no ring slot reloaded and no TMEM region overwritten before
its last reader)."""
import pytest

import bwd_protocol_model as bm

SHAPES = [dict(kv=True, dp_bufs=1), dict(kv=True, dp_bufs=2), dict(kv=False, dp_bufs=2)]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda c: f"kv{int(c['kv'])}-dp{c['dp_bufs']}")
@pytest.mark.parametrize("count", [1, 2, 3, 4, 7, 32])
def test_backward_protocol_runs_clean(shape, count):
    for seed in range(4):
        sim = bm.BwdSim(count, seed=seed, **shape)
        r = sim.run()
        assert r == "ok", (seed, r)
        assert not sim.errors, (seed, sim.errors[:3])


@pytest.mark.parametrize("flaw,dp_bufs", [("skip_sread", 1), ("early_a_empty", 1),
                                          ("shared_full", 2)])
def test_model_catches_a_broken_protocol(flaw, dp_bufs):
    """The model is not vacuous: issuing the next S before this step's S has
    been read, releasing an A-ring slot before dK / dQ has read it, or (with
    two dP regions, where a warp can run a step ahead) one P_FULL / DS_FULL
    barrier for every step, shows operands of the wrong step or a misread
    parity in some schedule."""
    bad = 0
    for seed in range(20):
        sim = bm.BwdSim(32 if flaw == "shared_full" else 8, kv=True, dp_bufs=dp_bufs, seed=seed,
                        **{flaw: True})
        r = sim.run()
        bad += (r != "ok") or bool(sim.errors)
    assert bad > 0


UNITS = [[3, 1, 5, 2], [32, 32], [1, 1, 1, 1], [8, 7, 6, 5, 4, 3, 2, 1]]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda c: f"kv{int(c['kv'])}-dp{c['dp_bufs']}")
@pytest.mark.parametrize("units", UNITS, ids=lambda u: "-".join(map(str, u)))
def test_persistent_units_run_clean(shape, units):
    """A persistent CTA takes several (key or query block) units in turn: the
    next unit's resident tiles load once the last S / dP of this one have
    ended; its first S follows this unit's last dK / dQ, which waited for
    every warp to finish the last step; its first accumulating product
    follows every warp's epilogue read of the accumulators through that
    warp's P / dS arrivals for the new unit."""
    for seed in range(4):
        sim = bm.BwdSim(units, seed=seed, **shape)
        r = sim.run()
        assert r == "ok", (seed, r)
        assert not sim.errors, (seed, sim.errors[:3])


def test_model_catches_resident_tiles_reloaded_too_early():
    """Negative control: loading the next unit's resident tiles without
    waiting for the last S / dP products of this one to end shows an S or dP
    reading the wrong unit's tile in some schedule."""
    bad = 0
    for seed in range(20):
        sim = bm.BwdSim([4, 4, 4], kv=True, dp_bufs=1, seed=seed, skip_res_empty=True)
        r = sim.run()
        bad += (r != "ok") or bool(sim.errors)
    assert bad > 0
