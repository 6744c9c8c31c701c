"""fp64 CPU oracle for the TwELL gated FFN — test infrastructure only.

Only the tests, the smoke check and the benchmark's CPU-baseline leg import this
package. The product path never does.
"""
