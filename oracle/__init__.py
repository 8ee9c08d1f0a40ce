"""CPU oracle (float64, test infrastructure only; see ref.py)."""
