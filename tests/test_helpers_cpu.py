"""The acceptance helpers of the GPU parity tests, checked on the CPU.

width_is_near_tie decides whether a kept width found on the GPU may differ
from the one the oracle's rule gives on the oracle's own scores; it must
accept a cut that sits on tau * E within the window and reject any other.
"""
import numpy as np

from tests.helpers import ADAPTIVE_ENERGY_REL, width_is_near_tie


def test_width_near_tie_accepts_a_cut_on_the_threshold():
    # squared scores 4, 3, 2, 1 (E = 10): with tau = 0.7 the cumulative energy
    # 7 after two channels equals tau * E exactly, so widths 2 and 3 both follow
    # from scores perturbed within the tolerance
    s = np.sqrt(np.array([4.0, 3.0, 2.0, 1.0]))
    assert width_is_near_tie(s, 0.7, 1, 4, 2, 3)
    assert width_is_near_tie(s, 0.7, 1, 4, 3, 2)
    # just inside and just outside the window
    tau_in = 0.7 * (1 + 0.5 * ADAPTIVE_ENERGY_REL)
    tau_out = 0.7 * (1 + 3 * ADAPTIVE_ENERGY_REL)
    assert width_is_near_tie(s, tau_in, 1, 4, 2, 3)
    assert not width_is_near_tie(s, tau_out, 1, 4, 2, 3)


def test_width_near_tie_rejects_distant_widths():
    s = np.sqrt(np.array([4.0, 3.0, 2.0, 1.0]))
    assert not width_is_near_tie(s, 0.5, 1, 4, 1, 3)   # cum 4 and 7 are far from 5
    assert not width_is_near_tie(s, 0.7, 1, 4, 1, 3)   # cum 4 is far from 7
    assert not width_is_near_tie(s, 0.7, 3, 4, 2, 3)   # a width below T_min cannot occur
