"""CPU check that the rescale case of the GPU attention tests does what it is for:
with the standard weights no query row ever rescales its running output, and with
the self-attention Q/K weights doubled many rows do, at different key tiles, so the
rows of one 32-row warp disagree (in whole items, and in the split schedule of 296
persistent CTAs that a 148-SM B200 takes at 64x64x640)."""
import pytest

from rescale_case import CASES, divergent_events


def test_standard_weights_never_rescale():
    assert divergent_events(48, 48, 320, None, qk_scale=1.0) == (0, 0)


@pytest.mark.parametrize("H,W,C,ctas", CASES)
def test_doubled_qk_makes_warp_rows_disagree(H, W, C, ctas):
    events, divergent = divergent_events(H, W, C, ctas)
    assert divergent > 100, (events, divergent)
