"""CPU oracle (test infrastructure only; see tb_oracle.py)."""
