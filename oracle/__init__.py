"""fp64 CPU oracle of RecSA (test infrastructure only; see recsa_oracle.py)."""
