"""Measurement command lines beside bench.py: equal-cost prefill chunking (chunking), attention
recall and budget sweeps (recall) and the decode step (decode_bench). Each runs the library
through its C ABI on the seeded synthetic workloads and prints JSON."""
