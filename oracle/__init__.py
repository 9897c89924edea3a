"""CPU oracle (test infrastructure only): a plain fp64 restatement of the sparse decode step."""
