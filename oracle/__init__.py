"""CPU oracle of the HSA hot path: test infrastructure only (see hsa_oracle.py)."""
