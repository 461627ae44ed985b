"""B200-native sketched linear layer (SpaLLM / SketchTune LUT path).

The compute lives in ``libsk.so`` (C ABI, hand-written sm_100a kernels); the
Python binding in ``compressive_fine_tuning_b200.sk`` only marshals arguments.
``synth`` draws seeded synthetic inputs.  Importing the package itself loads
nothing native; ``import compressive_fine_tuning_b200.sk`` does.
"""

__all__ = ["sk", "synth", "build"]
