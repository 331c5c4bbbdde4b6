"""Plain, slow CPU oracle (fp64) for the block-diffusion denoising step.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline and reference legs of ``bench.py`` may import it.

* ``step.cc``: the oracle, a plain C++ program (naive loops, fp64, no BLAS,
  ``std::thread`` over independent heads, vocabulary ranges and rows), built
  by ``build.py`` into ``liboracle.so``; ``step.py`` is its ctypes binding.
* ``step_np.py``: an independent numpy restatement of the same definitions,
  used only as a second check of the C++ program.
* ``theory.py``: the joint-distribution mathematics behind the selection
  rules (pins of the theorem); ``cases.py``: margin-repaired parity cases.

It shares no code with the CUDA library; the only shared module is the
seeded input generator (``block_diffusion_decoding_causal_b200.synth``),
which holds none of the method's arithmetic.

Parity unpinned: the point at which the attention output is rounded to bf16
before it feeds the LM head, and the GPU's fp32 exponentials.  The pages fix
neither; the parity tolerances and the decision margins of ``cases`` cover
both.
"""
