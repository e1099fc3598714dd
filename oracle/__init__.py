"""fp64 CPU oracle for the DiT joint-attention hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or links
this package: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.  It shares no code with the CUDA path; its inputs
come from the seeded generators in ``diffusion_transformer_denoising_dit_b200.synth``
(which hold no arithmetic of the method) or are built by the tests.

Every function is a plain, slow restatement of a definition, in numpy float64,
one step at a time.  Sources (the pages these definitions are read from):

* [VisualGen] "FLUX 3 Image Klein / TensorRT-LLM VisualGen" (devotd.net news),
  section "why the differences arise": BF16 "VANILLA" attention is about 60 %
  of DiT GPU kernel time; cuDNN FP8 attention; Cache-DiT residual threshold.
* [FBCache] unsloth studio commit "core/inference/diffusion.py", paragraph
  "Add opt-in step caching (First-Block-Cache)": skip the remaining blocks once
  the first block's residual barely changes.
* [vflash] "vflash / Optimization ledger", table "Accepted or exposed":
  SageAttention2 (quantised attention) and strict Triton RoPE.

None of the pages writes down a formula for attention, rotary embedding, K
smoothing, FP8 block quantisation or the cache residual test; the definitions
here are the textbook ones those names denote, and each reading the pages leave
open is stated where it is used.

Parity status: attention, RoPE, the e4m3 quantiser and the gate are pinned by
closed forms, invariants, brute force and independent library special cases
(tests/test_oracle_*.py).  ``fp8.simulated_attention`` is a diagnostic of our
own reading of an unspecified quantised scheme: the reading cannot be pinned to
the pages, its implementation is pinned by closed forms and invariants of that
reading (and planted mistakes fail them).
"""
from . import attention, fp8, gate, rope  # noqa: F401
