"""fp64 CPU oracle for KDA -- test infrastructure only (see kda_oracle.py)."""
