"""CPU oracle package -- test infrastructure only (see oracle/oracle.py and oracle/kvk_oracle.c)."""
