"""CPU oracle for the grouped sparse-NVFP4 expert GEMM path.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package.  The library never does,
and nothing here imports the library: the two share no code.  Inputs reach both
sides from ``grouped_sparse_gemm_b200.inputs``, which only draws random numbers.

What it computes comes from "Hardware-Native Joint Sparse-Quantization for
Trillion-Scale Mixture-of-Experts" (paperlayer.ai summary page): paired 4:8
sparsity with E2M1 values and one UE4M3 scale per 32 logical weights (App. A,
pp.14-15), NVFP4 activations in 32-element blocks fused with dispatch (§D.1),
and grouped execution of the routed expert products with the sparse weight as
operand A (§3.4), and the SwiGLU output preparation between the two expert GEMMs (§D.1).
Every step is the plain definition, in numpy (float32 where
the step is an fp32 operation, float64 for the reference products).

Pins (tests/test_oracle_*.py): exhaustive code tables, rounding midpoints,
brute force over the six pair patterns, round trips on representable weights,
closed forms for the GEMM, the 2.75 bit/weight count, routing invariants and a
hand-worked golden example under tests/golden/.  Nothing here is "parity
unpinned".
"""
from . import codecs, pack, quant, route, gemm, unpermute, layout, swiglu  # noqa: F401

__all__ = ["codecs", "pack", "quant", "route", "gemm", "unpermute", "layout", "swiglu"]
