"""CPU oracle for NSNQuant encode / dequant / decode attention (test infrastructure only)."""
