"""B200-native SuperGlue matcher forward pass: C-ABI library ``libsg`` plus a thin
ctypes binding.  ``synth`` holds the seeded synthetic workloads."""
__version__ = "0.1.0"
