import os
import sys

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
"""Race detection for the attention kernel's barrier protocol (CPU): the
model in protocol_model.py runs the kernel's roles under random timings with
warp drift and a tensor pipe that may complete UMMA groups in any order.  The
shipped protocol must show no parity aliasing, no conflicting TMEM/shared
memory access and no deadlock; two earlier, racy designs must be caught."""
import pytest

from protocol_model import ProtocolError, simulate, simulate_gemm, simulate_gemm_pair


@pytest.mark.parametrize("n_items,n_kt", [(1, 1), (2, 1), (3, 2), (4, 3), (2, 7)])
def test_shipped_protocol_is_race_free(n_items, n_kt):
    for seed in range(60):
        simulate(seed, n_items=n_items, n_kt=n_kt)


@pytest.mark.parametrize("n_items,n_kt", [(2, 1), (4, 3)])
def test_split_score_protocol_is_race_free(n_items, n_kt):
    # an alternative issue order (measured slower, not shipped): the first
    # half of S(k + 3) queued behind PV(k), P over columns 64..127
    for seed in range(30):
        simulate(seed, n_items=n_items, n_kt=n_kt, split_s=True)


def test_checker_catches_p_over_the_half_the_early_scores_overwrite():
    # split S with P written over columns 0..63: S(k + 3)'s first half would
    # overwrite P while PV(k) reads it
    import protocol_model as pm

    caught = 0
    old = pm.P_HALF
    pm.P_HALF = 0
    try:
        for seed in range(100):
            try:
                simulate(seed, n_items=3, n_kt=2, split_s=True)
            except ProtocolError:
                caught += 1
    finally:
        pm.P_HALF = old
    assert caught > 0


@pytest.mark.parametrize("n_items,n_kt,splits", [(3, 2, (True, False, True)), (4, 3, (False, True, True, False)),
                                                  (2, 1, (True, True)), (5, 7, (False,) * 4 + (True,)),
                                                  (6, 2, (False, False, True, False, False, True))])
def test_split_items_are_race_free(n_items, n_kt, splits):
    # items whose two tiles straddle two units stream K/V per warpgroup
    for seed in range(25):
        simulate(seed, n_items=n_items, n_kt=n_kt, splits=splits)


@pytest.mark.parametrize("n_items,n_kt,splits", [(1, 1, ()), (3, 1, ()), (4, 3, (False, True, False, True)),
                                                  (5, 2, (True,) * 5), (2, 11, (False, True))])
def test_deferred_epilogue_is_race_free(n_items, n_kt, splits):
    # the general kernel: an item's epilogue inside the next item's first step
    for seed in range(25):
        simulate(seed, n_items=n_items, n_kt=n_kt, splits=splits, defer_epilogue=True)


def test_checker_catches_the_deferred_epilogue_after_p_ready():
    caught = 0
    for seed in range(100):
        try:
            simulate(seed, n_items=4, n_kt=1, defer_epilogue=True, mutation="defer_after_ready")
        except ProtocolError:
            caught += 1
    assert caught > 0


def test_checker_catches_split_items_released_as_shared():
    caught = 0
    for seed in range(200):
        try:
            simulate(seed, n_items=4, n_kt=3, splits=(False, True, False, True), mutation="split_shared_release")
        except ProtocolError:
            caught += 1
    assert caught > 0


@pytest.mark.parametrize("mutation", ["single_p_ready", "epilogue_o_done"])
def test_checker_catches_the_earlier_races(mutation):
    caught = 0
    for seed in range(200):
        try:
            simulate(seed, n_items=4, n_kt=3, mutation=mutation)
        except ProtocolError:
            caught += 1
    assert caught > 0, f"{mutation}: the race was never detected"


@pytest.mark.parametrize("n_tiles,k_chunks", [(1, 1), (3, 2), (8, 5), (5, 16)])
def test_gemm_protocol_is_race_free(n_tiles, k_chunks):
    for seed in range(60):
        simulate_gemm(seed, n_tiles=n_tiles, k_chunks=k_chunks)


def test_checker_catches_an_accumulator_reused_before_the_epilogue_read_it():
    caught = 0
    for seed in range(100):
        try:
            simulate_gemm(seed, mutation="no_acc_empty")
        except ProtocolError:
            caught += 1
    assert caught > 0


@pytest.mark.parametrize("n_tiles,k_chunks", [(1, 1), (3, 2), (8, 5), (5, 16)])
def test_gemm_pair_protocol_is_race_free(n_tiles, k_chunks):
    for seed in range(25):
        simulate_gemm_pair(seed, n_tiles=n_tiles, k_chunks=k_chunks)


@pytest.mark.parametrize("mutation", ["pair_follower_expects", "pair_commit_leader_only", "pair_local_release"])
def test_checker_catches_pair_protocol_mistakes(mutation):
    caught = 0
    for seed in range(15):
        try:
            simulate_gemm_pair(seed, n_tiles=5, k_chunks=8, mutation=mutation)
        except ProtocolError:
            caught += 1
            break
    assert caught > 0, f"{mutation}: never detected"
