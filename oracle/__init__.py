"""Float64 CPU oracle for the online long-convolution mixer stack.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports, calls, links or
executes anything in this package: only the test suite, the package smoke check
and the benchmark's CPU-baseline leg use it. It shares no code with the CUDA
library; both sides receive the same arrays from the seeded input generator.

Source of every definition: "Flash Inference: Near Linear Time Inference for Long
Convolution Sequence Models and Beyond" (Oncescu, Purandare, Idreos, Kakade;
arXiv 2410.12982), as summarised on the lowest.today article page. Sections are
cited by that page's (Italian) headings.

Pins: every function here is pinned by tests under ``tests/test_oracle*.py`` to
something other than itself (library routines, closed forms, invariants, brute
force, the schedule facts the page prints).
"""
from .lcsm import (  # noqa: F401
    bf16_round,
    causal_conv,
    causal_conv_at,
    dft,
    gelu,
    lowbit,
    mlp_block,
    online_lcsm,
    online_lcsm_mlp,
    prompt_lcsm,
    relaxed_online,
    relaxed_tiles,
    stream_error,
    tau,
)
