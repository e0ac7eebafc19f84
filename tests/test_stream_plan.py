"""The layer-visit schedule of a streamed step (host logic, no GPU): lsq_stream_plan
returns the plan stream_stack_step follows.  Checked by replaying it against a
model of the two VRAM buffers."""
import ctypes
import os

import pytest

from layer_streamed_qlora_nf4_b200 import lib as L


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from layer_streamed_qlora_nf4_b200 import build
    if not os.path.exists(L.LIB_PATH):
        build.build()
    L.load()


def _replay(plan, L_, mb, held):
    """Checks every visit against the buffer contents; returns (copies, final contents)."""
    held = list(held)
    order = [k for _ in range(mb) for k in list(range(L_)) + list(range(L_ - 1, -1, -1))]
    assert [v[0] for v in plan] == order           # forward 0..L-1, backward L-1..0
    copies = 0
    for i, (layer, buf, copy) in enumerate(plan):
        assert buf in (0, 1)
        if copy:
            assert layer not in held                   # copied only when not resident
            if i > 0:                                  # never into the buffer the previous
                assert buf != plan[i - 1][1]           # visit is still computing on
            held[buf] = layer
            copies += 1
        else:
            assert held[buf] == layer                  # a reused buffer holds the layer
    return copies, tuple(held)


@pytest.mark.parametrize("n_layers", [1, 2, 3, 4, 5, 32])
@pytest.mark.parametrize("mb", [1, 2, 4])
def test_plan_replays_and_counts_copies(n_layers, mb):
    held = (-1, -1)
    counts = []
    for _ in range(3):                                 # three steps, contents carried over
        plan = L.lsq_stream_plan(n_layers, mb, *held)
        c, held = _replay(plan, n_layers, mb, held)
        counts.append(c)
    if n_layers == 1:
        assert counts == [1, 0, 0]
        return
    # first step: the forward->backward turn finds layers L-1 and L-2 resident; each later
    # micro-batch (and step) also finds layers 0 and 1 resident
    first = (2 * n_layers - 2) + (mb - 1) * max(0, 2 * n_layers - 4)
    steady = mb * max(0, 2 * n_layers - 4)
    assert counts == [first, steady, steady]
    assert sorted(held) == [0, 1]                      # a step ends holding layers 0 and 1


def test_plan_from_arbitrary_contents():
    for held in [(5, -1), (-1, 7), (3, 4), (31, 0)]:
        plan = L.lsq_stream_plan(32, 1, *held)
        _replay(plan, 32, 1, held)


def test_plan_argument_errors():
    with pytest.raises(L.LsqError) as e:
        L.lsq_stream_plan(0, 1)
    assert e.value.code == L.LSQ_ERR_SHAPE
    with pytest.raises(L.LsqError) as e:
        L.lsq_stream_plan(4, 1, 2, 2)                  # one layer in both buffers
    assert e.value.code == L.LSQ_ERR_SHAPE
    with pytest.raises(L.LsqError) as e:
        L.lsq_stream_plan(4, 1, 4, -1)                 # no such layer
    assert e.value.code == L.LSQ_ERR_SHAPE
    out = [(ctypes.c_int32 * 4)() for _ in range(3)]
    n = ctypes.c_int32(0)
    rc = L.load().lsq_stream_plan(4, 1, -1, -1, out[0], out[1], out[2], 4, ctypes.byref(n))
    assert rc == L.LSQ_ERR_WORKSPACE                   # 8 visits, room for 4
