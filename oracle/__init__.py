"""CPU oracle for the Muon step (float64 numpy).  Test infrastructure only:
see ``oracle.muon_oracle``."""

from .muon_oracle import (  # noqa: F401
    NS_A, NS_B, NS_C, NS_EPS, NS_STEPS,
    quintic, newton_schulz5, momentum_update, muon_update,
)
