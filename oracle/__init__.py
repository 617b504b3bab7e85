"""Plain fp64 CPU oracle for the SLA / SLA2 sparse-plus-linear block attention forward.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package. The product (the CUDA
library and its Python binding) never calls it and shares no code with it.

Everything here is written for a reader checking it against the pages, not for
speed: float64 throughout, the steps in the order the method states them, numpy
matmul/sort as the only library primitives.

Sources (page title, section):

* "SLA: Beyond Sparsity in Diffusion Transformers via Fine-Tunable
  Sparse-Linear Attention", Abstract: attention weights are split into
  critical (exact O(N^2) attention), marginal (O(N) linear attention) and
  negligible (skipped) parts.
* "SLA2: Sparse-Linear Attention with Learnable Routing and QAT",
  §1 item 1: the sparse branch is softmax re-normalised over its own keys;
  §2.A: O = alpha * O_s + (1 - alpha) * O_l;
  §2.B: the router pools adjacent Q and K tokens and ranks blocks from the
  compressed scores; hard top-k at inference.
* "SPLA - Atención de Bloque Dispersa más Lineal para el Modelado de Contexto
  Largo", §2.1 (mean pooling of a block as its compressed key).

Readings where the pages are silent (each is listed with its reason in the
design notes):

* feature map phi(x) = elu(x) + 1, on raw q and k (no 1/sqrt(D));
* pooling = arithmetic mean over the valid tokens of a block;
* compressed score S_ij = qbar_i . kbar_j / sqrt(D); learned router
  projections are the identity; ranking uses S (softmax is monotone);
* counts: kc = ceil(kh_ppm * Nk / 1e6), kn = floor(kl_ppm * Nk / 1e6) with
  kh_ppm = round(kh * 1e6);
* per query-block row the total order is (S descending, j ascending); the
  first kc blocks are critical, the last kn negligible, the rest marginal;
* an empty critical set gives O_s = 0, an empty marginal set gives O_l = 0;
* alpha is [H, D], shared over batch and tokens.
"""

from .sla_oracle import (  # noqa: F401
    block_counts,
    phi,
    pool_mean,
    compressed_scores,
    compressed_probs,
    route,
    route_from_scores,
    kv_states,
    sparse_branch,
    marginal_sums,
    linear_branch,
    forward,
    as_f64,
)
