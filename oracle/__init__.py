"""CPU oracle for the MXCode W4A4 linear layer (test infrastructure; see mxcode_oracle)."""
