"""persistent_megakernel_03_b200: batch-1 transformer decode as one persistent
sm_100a megakernel (task graph + event counters + TMA weight ring).

The compute path is the C-ABI library ``libmk.so`` (built from ``csrc/``);
``binding`` is its ctypes marshalling layer.  ``synth`` draws the seeded
synthetic models and prompts.  Importing this package loads nothing native;
``binding.lib()`` does, and fails loudly when the library is missing.
"""
__all__ = ["synth", "binding"]
