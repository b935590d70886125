"""Position maps from the CUDA library, bit-exact against the oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from position_remapping_b200.inputs import MapParams

pytestmark = pytest.mark.gpu

CASES = [
    MapParams(O.STANDARD),
    MapParams(O.NOPE),
    MapParams(O.ENDPROMPT, rope_base=5e5, interp=8.0, seg1_len=8000, term_start=65344),
    MapParams(O.ENDPROMPT, seg1_len=0, term_start=12345),
    MapParams(O.PERIODIC, window=1024),
    MapParams(O.PERIODIC, window=1),
    MapParams(O.PERIODIC, window=64),
    MapParams(O.BIFOCAL, rope_base=1e6, w0=2048, w_pretrained=32768),
    MapParams(O.BIFOCAL, rope_base=1e6, w0=0, w_pretrained=3),
]
LENGTHS = [1, 2, 127, 128, 129, 8192, 32767, 32768, 32769, 65536, 65537, 98304, 131072, 131073]


@pytest.mark.parametrize("params", CASES, ids=lambda p: f"kind{p.kind}")
def test_posmap_bit_exact(params):
    from position_remapping_b200 import ropeattn as ra
    for L in LENGTHS:
        loc, rem, G = ra.posmap(params, L)
        torch.cuda.synchronize()
        want_loc, want_rem, want_G = O.position_maps(params, L)
        assert G == want_G, (L, G, want_G)
        assert np.array_equal(loc.cpu().numpy().astype(np.int64), want_loc), L
        if params.kind == O.BIFOCAL:
            assert np.array_equal(rem.cpu().numpy().astype(np.int64), want_rem), L
            assert int(rem.max()) <= params.w_pretrained - 1


def test_posmap_empty_is_noop():
    from position_remapping_b200 import ropeattn as ra
    loc, rem, G = ra.posmap(CASES[7], 0)
    assert loc.numel() == 0 and G == 1
