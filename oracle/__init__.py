"""Float64 CPU oracle of the equivariant convolution.

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline / reference arm, never by the product path."""
from .core import (NORMALIZATIONS, Irrep, Path, Plan, backward, bessel_cutoff, cg, forward,
                   irreps_linear,
                   max_threads, parse_irreps, plan, radial_mlp, random_rotation, sh, sh_l, silu, wigner_3j,
                   wigner_d)

__all__ = ["NORMALIZATIONS", "Irrep", "Path", "Plan", "backward", "bessel_cutoff", "cg", "forward",
           "irreps_linear",
           "max_threads", "parse_irreps", "plan", "radial_mlp", "random_rotation", "sh", "sh_l",
           "silu", "wigner_3j", "wigner_d"]
