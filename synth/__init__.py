"""Seeded synthetic inputs for the routed mixture-of-experts FFN.

This package is the one piece shared by the float64 oracle and the CUDA path.
It draws numbers and lays out the self-defined block format's canonical
bytes; it holds none of the method's arithmetic (no dequantisation, routing,
FFN, combine or normalisation).

* ``rng``      SplitMix64 (Steele, Lea & Flood 2014; Vigna's reference
               implementation) as a counter-based generator, plus stream keys.
* ``configs``  the five synthetic workloads (shapes, formats, distributions).
* ``gen``      host generation of codes, fp16 (d, m) pairs and Gaussians.
* ``device``   ctypes binding of ``libqmoe_synth.so``, the same code and scale
               streams filled on the GPU (bit-identical to ``gen``).
"""
from . import configs, rng, gen  # noqa: F401
