"""CPU oracle package -- test infrastructure only (see s6_oracle.py)."""
