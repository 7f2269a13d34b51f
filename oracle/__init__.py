"""fp64 CPU oracle for blockwise causal varlen attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(the CUDA library and its Python binding) never imports it, and it imports
nothing from the product path: the two share no kernels, helpers, tables or
pre/post-processing.  Inputs reach both from :mod:`synth`.

Everything is plain NumPy in float64, written from the pages' statement of the
method (cited per function by page title and section):

* ``attention``  - exact masked softmax attention, its log-sum-exp, its analytic
  gradients, and the online-softmax merge of partial results;
* ``planner``    - the zig-zag / contiguous context-parallel layouts, half
  indices, halved cu_seqlens and per-rank work counts (integer, exact);
* ``ring``       - the zig-zag and contiguous ring loops over virtual ranks,
  block by block, merged with the log-sum-exp identity, and their backward
  fed the merged out/lse;
* ``paged``      - KV-parallel segmented prefill over a paged KV cache;
* ``decode``     - one-query-per-sequence GQA varlen decode;
* ``cached``     - EAGLE-3 cached attention: the causal sequence block plus the
  per-position cache diagonals in one softmax, and its analytic gradients.

Pins (tests marked ``not gpu``): brute force on tiny inputs, closed forms
(q = 0 gives lse = log|visible| and out = mean of visible values), finite
differences of the gradients, gradient sum rules, merge-order invariance,
integer work-balance formulas and the hand-derived planner example stored under
``tests/golden``.  Parity unpinned: none of the functions here is left without
an independent pin; the absolute values of out/lse/gradients on random inputs
rest on the definition itself, which the pins check term by term.
"""
