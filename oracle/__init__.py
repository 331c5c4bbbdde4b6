"""Plain, slow CPU oracle (fp64) for the block-diffusion denoising step.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import it.  It shares no code with the
CUDA library; the only shared module is the seeded input generator
(``block_diffusion_decoding_causal_b200.synth``), which holds none of the
method's arithmetic.

Parity unpinned: the point at which the attention output is rounded to bf16
before it feeds the LM head, and the GPU's fp32 exponentials.  The pages fix
neither; the parity tolerances and the decision margins of ``cases`` cover
both.
"""
