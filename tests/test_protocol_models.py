"""The kernels' barrier protocols, checked by randomised models (tests/pba_protocol_models.py):
many interleavings per configuration, ring and buffer depths as the kernels instantiate them,
and planted mistakes that the checks must catch."""
import pytest

from pba_protocol_models import BwdSim, DbiasSim, FwdSim, PwaGemmSim


# ring depths as the forward instantiates them: c=16 -> (3, 2), c=32 -> (2, 2), c=64 -> (2, 1)
@pytest.mark.parametrize("KVS,BS", [(2, 2), (3, 2), (2, 1)])
def test_forward_protocol(KVS, BS):
    # items of nb rows over nJ key tiles (the last chunk of rows can be shorter)
    for nJ in (1, 2, 3):
        for nbs in ([1], [2, 2], [2, 1], [4, 4, 3], [1, 1, 1, 1]):
            for row_mask in (False, True):
                for seed in range(12):
                    FwdSim(nJ, nbs, KVS, BS, seed, row_mask).run()


# c=32 -> (2, 2, 2, 2), c=16 -> (3, 2, 2, 2), c=64 -> (2, 1, 1, 1); the last mixes depths
@pytest.mark.parametrize("QS,BS,KVB,DKB", [(2, 2, 2, 2), (3, 2, 2, 2), (2, 1, 1, 1), (2, 2, 1, 2)])
def test_backward_protocol(QS, BS, KVB, DKB):
    # items with a fixed or a varying number of steps (local attention)
    for M in (0, 1, 2, 3, 5):
        for nI in (1, 2, 3, [1 + (m * 7 + 3) % 3 for m in range(M)]):
            for seed in range(12):
                BwdSim(M, nI, QS, BS, KVB, DKB, seed).run()


def _caught(make, seeds=40):
    for seed in range(seeds):
        try:
            make(seed).run()
        except (AssertionError, RuntimeError):
            return True
    return False


def test_planted_forward_mistake_is_caught():
    # Q of the next item loaded before the previous item's last Q K^T is done
    assert _caught(lambda seed: FwdSim(2, [2, 2, 2], 2, 2, seed, plant="no_q_empty_wait"))


def test_planted_backward_mistakes_are_caught():
    # P/dS rewritten before the previous step's products are done
    assert _caught(lambda seed: BwdSim(4, 2, 2, 2, 2, 2, seed, plant="no_ps_free_wait"))
    # a dK/dV accumulator reused before its epilogue has read it (one buffer, one step per item)
    assert _caught(lambda seed: BwdSim(4, 1, 2, 2, 2, 1, seed, plant="no_dkv_free_wait"))
    # with one K/V stage, S/dP of an item's first step issued before the previous item's last
    # dQ, which is what frees the stage: deadlock
    assert _caught(lambda seed: BwdSim(3, 2, 2, 1, 1, 1, seed, plant="sdp_before_dq"))


# dbias kernel stages: c=64 -> 2, otherwise 3
@pytest.mark.parametrize("NS", [2, 3, 5, 8])
def test_dbias_protocol(NS):
    for nb in (0, 1, 2, 3, 4, 7):
        for seed in range(40):
            DbiasSim(nb, NS, seed).run()


def test_planted_dbias_mistakes_are_caught():
    # a stage refilled before the MMA and both warpgroups are done with it
    assert _caught(lambda seed: DbiasSim(6, 2, seed, plant="no_empty_wait"))
    # S/dP of row n + 2 issued into the TMEM buffer row n is still read from (with two stages
    # the stage's own empty barrier happens to cover this; with three it does not)
    assert _caught(lambda seed: DbiasSim(6, 3, seed, plant="no_sd_free_wait"))


# GEMM: 2 stages; dW: 4 stages (and possibly no rows in a split)
@pytest.mark.parametrize("NS", [2, 4])
def test_pwa_gemm_protocol(NS):
    for nK in (0, 1, 2, 3, 4, 5, 9):
        for seed in range(40):
            PwaGemmSim(nK, NS, seed).run()


def test_planted_pwa_gemm_mistakes_are_caught():
    assert _caught(lambda seed: PwaGemmSim(5, 2, seed, plant="no_empty_wait"))
    # the epilogue signalled before the last products are done
    assert _caught(lambda seed: PwaGemmSim(5, 2, seed, plant="early_done"))
