"""B200-native GPTQ layer solver: a C-ABI CUDA library (``libgptq.so``) and a thin binding.

Importing the package does not load the library; ``post_weight_quantization_20_b200.gptq``
loads it on first use and fails loudly if it has not been built.
"""
