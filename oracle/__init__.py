"""CPU oracle (float64, numpy) for the AWQ search path. Test infrastructure only."""
