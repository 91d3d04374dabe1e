"""Host logic of the parity helpers (no GPU): the tie-band split of a unit's
candidates and the check that a selection is one of the valid top-k sets."""
import numpy as np
import pytest

from parity import band_parts, valid_choice


def unit_scores():
    # candidates 2..9 (NaN elsewhere); pages 4 and 7 tie inside the band
    sc = np.full(12, np.nan)
    sc[2:10] = [5.0, 9.0, 7.0, 1.0, 3.0, 7.0 + 1e-6, 8.0, 0.5]
    return sc


def test_band_parts_splits_must_and_band():
    sc = unit_scores()
    must, band = band_parts(sc, 3)          # top: 3 (9), 8 (8), then 4 / 7 (7, 7+1e-6)
    assert must == {3, 8} and band == {4, 7}
    must, band = band_parts(sc, 2)          # gap 9 -> 8 -> 7 is wide: no band
    assert must == {3, 8} and band == set()
    assert band_parts(sc, 0) == (set(), set())
    must, band = band_parts(sc, 8)          # every candidate
    assert must == set(range(2, 10)) and band == set()


def test_valid_choice_accepts_a_band_pick_and_rejects_others():
    sc = unit_scores()[None, None, :]
    ref_sel = np.array([[[3, 7, 8]]], np.int32)     # the oracle's own (page 7 scores higher)
    ref_nsel = np.array([[3]], np.int32)
    sel, nsel, same = valid_choice(ref_sel, ref_nsel, sc, ref_sel, ref_nsel)
    assert same == 1 and sel[0, 0, :3].tolist() == [3, 7, 8]
    pick = np.array([[[3, 4, 8]]], np.int32)        # the other page of the band: valid
    sel, nsel, same = valid_choice(pick, ref_nsel, sc, ref_sel, ref_nsel)
    assert same == 0 and sel[0, 0, :3].tolist() == [3, 4, 8] and nsel[0, 0] == 3
    with pytest.raises(AssertionError):             # a page below the band
        valid_choice(np.array([[[2, 3, 8]]], np.int32), ref_nsel, sc, ref_sel, ref_nsel)
    with pytest.raises(AssertionError):             # misses a page above the band
        valid_choice(np.array([[[3, 4, 7]]], np.int32), ref_nsel, sc, ref_sel, ref_nsel)
    with pytest.raises(AssertionError):             # wrong count
        valid_choice(ref_sel, np.array([[2]], np.int32), sc, ref_sel, ref_nsel)
