"""CPU oracle of the weight fake-quantizer: test infrastructure only.

Only the tests, the smoke check and the benchmark's CPU baseline leg may
import this package. The product path (the CUDA library and its Python
binding) never does, and shares no code with it.
"""
