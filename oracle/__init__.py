"""Plain, slow fp64 CPU oracle for the QJL / FQJL key-sketch hot path.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package. The CUDA library never calls it, and it shares no code with the CUDA
library: no kernels, headers, helpers, tables or constants. Its random-number
generator is written here, separately, from the published definition of
Philox4x32-10.

Sources (web pages; each function cites the passage it follows):

* "Majid Daliri" author page (scholarfeed), abstract of QJL by Zandieh, Daliri
  and Han. It covers the JL transform followed by sign-bit quantisation, the
  absence of stored quantisation constants, and the asymmetric estimator in
  which one vector is sketched and the other is only JL-projected.
* "Fast Quantized Johnson - Lindenstrauss Transforms" (AI Radio episode page).
  Its sections "In short", "Key concepts", "The paper" (abstract) and
  "Transcript: The paper's improvements" cover D-FQJL and P-FQJL. Both are
  compositions of two randomized Hadamard transforms with a Gaussian second
  diagonal, and either Gaussian dither before the sign (D) or a random
  permutation between the two Hadamard stages (P).
* "Vladimir Braverman" author page (catalyzex), abstract "KIVI: A Tuning-Free
  Asymmetric 2bit Quantization for KV Cache". It covers per-token 2-bit value
  quantisation and the decode step that reads the whole KV cache per token.

Modules:
    philox     counter-based generator (Salmon et al., SC'11), uniforms, Box-Muller
    params     projection parameters drawn from a seed (dense S; D_r, Pi, D_g; dither)
    hadamard   Sylvester Hadamard matrix
    qjl        key sketch, query projection, asymmetric estimator
    kivi       2-bit per-token value quantisation
    attention  softmax(scores) . V over dequantised values
    paged      append one token per group into pages; reads through a block table

Parity status (each function's pins are in tests/test_oracle_*.py):
    Every function is pinned. The generator's bit stream is pinned by the
    published Philox4x32-10 known-answer vectors, and by its statistics; see
    ``philox``.
"""

from . import philox, params, hadamard, qjl, kivi, attention, paged  # noqa: F401
