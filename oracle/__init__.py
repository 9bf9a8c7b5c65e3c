"""CPU oracle for the rotated, quantized linear layer -- TEST INFRASTRUCTURE ONLY.

This package is the slow, obviously correct reference that the CUDA library is checked
against. It is plain NumPy in float64 and follows the definitions on the pages step by step:
dense block-Hadamard matrices instead of butterflies, a dense integer GEMM through fp64 BLAS,
a Lloyd iteration for the codebook. It shares no code with the CUDA library and imports
nothing from it; the library does not import it either.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import or run anything in here. The product path never falls back
to it.

Sources (pages are cited by title and section):
- OrbitQuant PR #25 ("Default changes" table; "Runtime work"): RPBH pre-rotation, the
  second independent RPBH round, absmax INT8 at A8, Lloyd-Max codebooks.
- CentriQ: Calibration-Free Quantization of Diffusion Transformers via Exact Mean Centering
  (§3 "Quantizers", Eq. 1; "Hadamard rotation", Lemma 1; §4.2 "Centering and exact
  re-injection", Eq. 4, Eq. 5, Eq. 6; "Scale and grid"; App. B.1, B.2 Eq. 9, B.3 Tab. 3;
  App. C.5 "Exactness").
- FLUX.1-schnell-OrbitQuant-W4A4 model card ("Quantization" settings: activation
  normalization epsilon 1e-10, rotation rpbh, rotation seed 0, block-size policy).

Parity status per function is listed in each module header.
"""
from .rpbh import (splitmix64_at, rpbh_plan, sylvester_hadamard, rotate, unrotate,
                   rpbh_matrix, default_block, default_rounds)
from .lloyd_max import (lloyd_max_gaussian, lloyd_max_gaussian_8bit, lloyd_max_mse,
                        lloyd_max_sphere, sphere_marginal)
from .quant import (EPS, PCT_RHO, PCT_GAMMA, center, absmax_quantize, lloyd_max_quantize,
                    percentile_quantize, pack_nibbles, unpack_nibbles, pack_pairs,
                    unpack_pairs)
from .linear import (quantize_activations, prepare_weights, gemm_int, gemm_lloyd_max,
                     epilogue, linear_forward, linear_unquantized)

__all__ = [
    "splitmix64_at", "rpbh_plan", "sylvester_hadamard", "rotate", "unrotate", "rpbh_matrix",
    "default_block", "default_rounds", "lloyd_max_gaussian", "lloyd_max_gaussian_8bit",
    "lloyd_max_mse", "lloyd_max_sphere",
    "sphere_marginal", "EPS", "center",
    "absmax_quantize", "lloyd_max_quantize", "percentile_quantize", "PCT_RHO", "PCT_GAMMA",
    "pack_nibbles", "unpack_nibbles", "pack_pairs", "unpack_pairs",
    "quantize_activations", "prepare_weights", "gemm_int", "gemm_lloyd_max", "epilogue",
    "linear_forward", "linear_unquantized",
]
