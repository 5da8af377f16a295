"""CPU oracle (test infrastructure only; see gdr_oracle.py). The product path never imports it."""
