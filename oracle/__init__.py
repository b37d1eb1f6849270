"""CPU oracle (test infrastructure only): see oracle/semkv_oracle.py."""
