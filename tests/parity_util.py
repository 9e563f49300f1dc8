"""The parity rules of the CUDA path against the oracle live beside the oracle
(oracle/parity.py, test infrastructure); the tests import them from here."""
from oracle.parity import (OUT_TOL, TIE_REL, W_ATOL, W_RTOL, check_parity, check_routing,  # noqa: F401
                           oracle_candidates, rel_gap)
