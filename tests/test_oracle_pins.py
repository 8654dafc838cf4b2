"""The CPU oracle against its pins (no GPU)."""
import pytest

import oracle
import pins


@pytest.fixture(scope="module")
def orc():
    return oracle.get()


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_rejects_bad_arguments(orc):
    import numpy as np
    with pytest.raises(ValueError):
        orc.fwd(np.ones((1, 2, 1)), np.ones((1, 2, 1)), np.ones((1, 0)), np.ones((1, 2, 0)),
                np.ones((1, 2, 0)))


def test_fp32_timing_build_tracks_the_oracle():
    """The fp32-accumulate build (a timed CPU baseline only) runs the same
    forward loop in single precision: it must agree with the fp64 oracle to
    fp32 accuracy on a seeded workload, with every option on."""
    import numpy as np

    from selective_state_space_31_b200 import synth
    inp = synth.make_fwd(2, 300, 8, 16, in_dtype="f32", seed=5, has_h0=True)
    kw = dict(D=inp.Dskip, z=inp.z, delta_bias=inp.delta_bias, h0=inp.h0)
    y64, h64 = oracle.get().fwd(inp.x, inp.delta, inp.A, inp.B, inp.C, **kw)
    y32, h32 = oracle.get_fp32().fwd(inp.x, inp.delta, inp.A, inp.B, inp.C, **kw)
    assert np.max(np.abs(y32 - y64)) / np.max(np.abs(y64)) < 1e-5
    assert np.max(np.abs(h32 - h64)) / np.max(np.abs(h64)) < 1e-5
    assert not np.array_equal(y32, y64)   # it really computes in fp32


def test_fwd_blocks_covers_every_channel():
    """The threaded block runner of the oracle gives the same values as one
    call over the whole problem."""
    import threading

    import numpy as np

    from selective_state_space_31_b200 import synth
    inp = synth.make_fwd(3, 50, 20, 8, in_dtype="f32", seed=6, has_h0=True)
    kw = dict(D=inp.Dskip, z=inp.z, delta_bias=inp.delta_bias, h0=inp.h0)
    y, h = oracle.get().fwd(inp.x, inp.delta, inp.A, inp.B, inp.C, **kw)
    gy, gh = np.full_like(y, np.nan), np.full_like(h, np.nan)
    lock = threading.Lock()

    def put(blk, yb, hb):
        b, d0, d1 = blk
        with lock:
            gy[b, :, d0:d1] = yb
            gh[b, d0:d1] = hb

    oracle.fwd_blocks(inp.x, inp.delta, inp.A, inp.B, inp.C, oracle.channel_blocks(3, 20, 7),
                      put, threads=4, **kw)
    assert np.array_equal(gy, y) and np.array_equal(gh, h)
