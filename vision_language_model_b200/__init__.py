"""B200-native image half of the Mistral 3 / Pixtral multimodal forward.

The compute path lives in the C-ABI library `libvlm_b200.so` (sm_100a CUDA
kernels); `vision_language_model_b200.vlm` is its thin ctypes binding and
`synth` draws the seeded synthetic inputs. Nothing here is imported eagerly:
importing the package does not load the library, the first call does, and it
raises if the library is missing.
"""
