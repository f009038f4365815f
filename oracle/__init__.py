"""CPU oracle (test infrastructure only): plain fp64 restatements of the encoder and the M-RoPE
index. Only tests, the smoke check and the benchmark's CPU leg may import this package."""
