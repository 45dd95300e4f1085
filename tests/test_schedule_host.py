"""Layer-schedule driver, host side (no GPU): the trunk builders follow the
stated readings, the workspace layout is the documented one, and every bad
descriptor or pointer is rejected before anything is queued."""
import ctypes

import pytest

from feed_forward_view_vggt_b200 import accounting, attn, schedules
from feed_forward_view_vggt_b200 import build as vbuild

N100 = attn.vggt_shape(100, 5, 37, 37, 16, 64)


@pytest.fixture(scope="module", autouse=True)
def built():
    vbuild.build()
    attn.load()


def test_vggt_trunk_alternates_frame_and_global():
    t = schedules.vggt_trunk(24)
    assert len(t) == 48
    assert t[0::2] == ["frame"] * 24 and t[1::2] == ["global"] * 24


def test_avggt_trunk_converts_the_early_third_and_subsamples_the_rest():
    t = schedules.avggt_trunk(24, stride=(2, 2))
    assert t[0::2] == ["frame"] * 24
    assert t[1:16:2] == ["frame"] * 8
    assert t[17::2] == [("sga", 2, 2)] * 16
    assert schedules.kind_counts(t) == {"frame": 32, ("sga", 2, 2): 16}
    assert schedules.kind_counts(schedules.avggt_trunk(6, converted=0, stride=(3, 3))) == \
        {"frame": 6, ("sga", 3, 3): 6}
    with pytest.raises(ValueError):
        schedules.avggt_trunk(4, converted=5)


def test_omega_trunk_turns_a_quarter_of_the_global_layers_into_register_attention():
    t = schedules.omega_trunk(24)
    glob = t[1::2]
    assert [i for i, x in enumerate(glob) if x == "register"] == [3, 7, 11, 15, 19, 23]
    assert schedules.kind_counts(t) == {"frame": 24, "global": 18, "register": 6}


def test_schedule_flops_add_up():
    N, ns, h, w, H, d = 100, 5, 37, 37, 16, 64
    L, S = ns + h * w, N * (ns + h * w)
    kept, dropped = accounting.sga_counts(N, ns, h, w, 2, 2)
    got = accounting.flops_schedule(schedules.avggt_trunk(24), N, ns, h, w, H, d)
    assert got == 32 * 4 * N * L * L * H * d + 16 * (4 * S * (kept + 1) * H * d + 4 * dropped * H * d)
    reg = accounting.flops_schedule(["register"], N, ns, h, w, H, d)
    assert reg == 4 * (N * ns) ** 2 * H * d


def _align(x):
    return (x + 255) // 256 * 256


def test_workspace_layout_is_the_documented_one():
    S = attn.vggt_num_tokens(N100)
    layers = ["frame", ("sga", 2, 2), "global", ("sga", 3, 3), ("sga", 2, 2), "register"]
    want = 0
    for s in ((2, 2), (3, 3)):
        want = _align(want + attn.vggt_sga_num_kept(N100, *s) * 4)
        want = _align(want + S * 4)
    want = _align(want + max(attn.vggt_sga_workspace_bytes(N100, 2, 2), attn.vggt_sga_workspace_bytes(N100, 3, 3)))
    assert attn.vggt_schedule_workspace_bytes(N100, layers) == want
    # no SGA layer: nothing to hold (register attention reads the specials in place)
    assert attn.vggt_schedule_workspace_bytes(N100, ["frame", "global", "register"]) == 0
    # repeating a stride does not grow the workspace
    one = attn.vggt_schedule_workspace_bytes(N100, [("sga", 2, 2)])
    assert attn.vggt_schedule_workspace_bytes(N100, [("sga", 2, 2)] * 7) == one


@pytest.mark.parametrize("layers", [[(7,)], [("sga", 0, 2)], [("sga", 2, -1)],
                                    [("sga", s, 1) for s in range(1, 10)]])
def test_bad_descriptors_give_no_workspace(layers):
    assert attn.vggt_schedule_workspace_bytes(N100, layers) == -1


def _call(layers, shape=N100, n=None, with_ptrs=False, workspace=None, ws_bytes=0, scale=0.125):
    lib = attn.load()
    n = len(layers) if n is None else n
    A = 1 << 28  # fake, aligned device addresses: never dereferenced on the paths tested here
    ptrs = (ctypes.c_void_p * max(n, 1))(*([A] * max(n, 1))) if with_ptrs else None
    return lib.vggt_attn_schedule(ptrs, ptrs, ptrs, ptrs, shape, attn._layers(layers), n, scale,
                                  workspace, ws_bytes, 0)


def test_schedule_rejects_bad_arguments_before_queuing():
    INVALID, WORKSPACE = attn.VGGT_ERR_INVALID_ARG, attn.VGGT_ERR_WORKSPACE
    assert _call([]) == attn.VGGT_OK                      # empty schedule: nothing to do
    assert _call([(9,)]) == INVALID                        # unknown kind
    assert _call([("sga", 0, 0)]) == INVALID               # bad stride
    assert _call([("sga", s, 1) for s in range(1, 10)]) == INVALID  # more than 8 strides
    assert _call(["frame"] * 1025) == INVALID                # more than VGGT_MAX_LAYERS
    no_specials = attn.vggt_shape(4, 0, 8, 8, 2, 64)
    assert _call(["register"], shape=no_specials) == INVALID
    assert _call(["frame"]) == INVALID                     # null pointer arrays
    assert _call(["frame"], with_ptrs=True, scale=0.0) == INVALID  # bad scale
    # frame/global only: no workspace is needed, so a null one is accepted;
    # the call then fails because o overlaps q (one fake address for all),
    # still before queuing anything
    assert _call(["frame"], with_ptrs=True) == INVALID
    assert _call(["frame"], with_ptrs=True, workspace=1 << 34, ws_bytes=0) == INVALID
    assert _call([("sga", 2, 2)], with_ptrs=True, workspace=1 << 34, ws_bytes=256) == WORKSPACE
    assert _call([("sga", 2, 2)], with_ptrs=True, workspace=(1 << 34) + 16, ws_bytes=1 << 40) == INVALID
