"""CPU oracle for the LLM.int8() decomposed linear layer -- test infrastructure only.

Only the test-suite, the smoke check and the CPU-baseline leg of the benchmark import
this package.  It shares no code with the CUDA library and imports nothing from it.
"""
