"""CPU float64 oracle (test infrastructure only; see ``oracle.ref``)."""
