"""KDA oracle (test infrastructure only; see kda_oracle.py)."""
