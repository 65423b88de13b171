"""B200-native weight-only-quantized mixture-of-experts forward (QMoE).

The compute path lives in ``csrc/`` (CUDA for sm_100a behind a C ABI,
declared in ``include/qmoe.h``); ``qmoe.py`` is its thin ctypes binding and
``inputs.py`` draws seeded synthetic inputs. Import ``qmoe`` explicitly; it
fails loudly when the compiled library is missing.
"""
