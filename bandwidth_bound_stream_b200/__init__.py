"""B200-native decode engine: one persistent sm_100a megakernel per GPU, driven through a
small C-ABI library (``libkie.so``, declared in ``include/kie.h``).

``kie`` is the Python binding (argument marshalling only); ``synth`` draws the seeded
synthetic weights and prompts. Nothing here imports the CPU oracle.
"""
