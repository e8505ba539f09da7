"""CPU oracle for the BASED hot path: Taylor linear attention and sliding-window attention.

THIS PACKAGE IS TEST INFRASTRUCTURE. Only the test suite, the smoke check in
``__graft_entry__`` and the ``cpu_baseline`` / reference leg of ``bench.py`` may
import it. The product path (the CUDA library and its Python binding) never
imports it and has no CPU fallback.

Everything here is plain, slow, float64 NumPy (plus pure-Python loops for the
brute-force cross-check on tiny inputs). It shares no code with the CUDA path:
no kernels, headers, helpers, tables or constants. Inputs arrive as float64
arrays holding the exact values the GPU sees (bf16-rounded where the GPU input
is bf16), so input quantisation is not counted as error.

Sources (all on the pages of "Simple linear attention language models balance
the recall-throughput tradeoff", BASED, arXiv 2402.18668v2, unless noted):

* linear attention through a feature map, with a recurrent form -- §2
  "Efficient attentions" and App. A.1;
* the 2nd-order Taylor feature map with projected dimension d' -- §4 "Taylor
  Linear Attention"; its explicit form phi(x) = [1, x, vec(x (x) x)/sqrt(2)],
  for which phi(q).phi(k) = 1 + q.k + (q.k)^2/2, is the problem statement this
  library is built to;
* the extra "K-state" z used for the denominator -- App. D.4 "State size";
* sliding-window softmax attention with a w-sized KV cache -- §4 "Local Exact
  Attention", App. A.1;
* the split of the output into order-0/1/2 Taylor terms and into an on-diagonal
  (causally masked, quadratic) and an off-diagonal (cumulative state) part --
  App. B "Forward / Generation Prefill" (Algorithm 1);
* the chunkwise form (intra-chunk + inter-chunk terms) -- "Gated Slot
  Attention", App. A.1 "Hardware-Efficient Training";
* the short gated convolution (BaseConv) mixer -- §4 "The BASED Architecture"
  (Additional mixers) and App. C "Extended Architecture Details" (Convolution).

Parity pins (see tests/test_oracle.py): closed forms, hand-derived golden
values, equivalence of independent formulations, textbook special cases, a
library softmax-attention routine, the O(eps^3) Taylor convergence to softmax
attention and pure-Python brute force on N <= 8. No page prints a worked
numeric example.
"""

from .taylor_la import (  # noqa: F401
    feature_map,
    feature_dim,
    la_quadratic,
    la_quadratic_parts,
    la_rows,
    la_state,
    la_recurrent,
    la_chunked,
    la_taylor_terms,
    packed_dim,
    packed_pairs,
    feature_map_packed,
    la_state_packed,
    la_recurrent_packed,
    la_backward,
    feature_map_vjp,
    la_backward_chunked,
    DECAY_CHUNK,
    decay_chunks,
    decay_per_step,
    decay_weights,
    la_quadratic_decay,
    la_recurrent_decay,
    la_state_decay,
)
from .swa import (  # noqa: F401
    swa,
    swa_rows,
    swa_ring_after_prefill,
    swa_decode_step,
)
from .baseconv import (  # noqa: F401
    silu,
    short_conv,
    baseconv,
    baseconv_state,
    baseconv_decode_step,
)
from . import brute  # noqa: F401
