"""Host-side argument checks of the overlapped step (no GPU needed)."""
import pytest


def test_overlapped_step_validates_before_touching_the_gpu():
    from muon_newton_schulz_05_b200.overlap import OverlappedStep
    with pytest.raises(ValueError):
        OverlappedStep([["bank"]], hp=None, variant="adamw")
    with pytest.raises(ValueError):
        OverlappedStep([], hp=None)
    with pytest.raises(ValueError):
        OverlappedStep([[], ["bank"]], hp=None)
