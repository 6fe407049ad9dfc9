"""KATA forward pass on B200 (sm_100a).

Causal normalized linear attention with the rank-one PSD feature map
psi(u) = vec(u u^T): o_t = sum_{s<=t} (q_t.k_s)^2 v_s / sum_{s<=t} (q_t.k_s)^2.

The computation lives in ``libkata.so`` (hand-written CUDA behind the C ABI of
``include/kata.h``); this package is its Python binding.  Entry points:

* :func:`kata_fwd_quadratic` -- flash-style O(T^2) forward;
* :func:`kata_fwd_chunked`   -- exact O(T) chunked-state forward with an
  associative scan across chunks;
* :func:`kata_decode_step`   -- one recurrent step on the fixed-size state;
* :func:`kata_fwd_chunked_noalloc` -- the chunked forward using a fixed
  library-owned scratch array, for callers that cannot allocate;
* :func:`kata_fwd_chunked_sequential` -- the sequential inter-chunk baseline
  (one CTA per sequence walks its chunks in order, no scan);
* :func:`kata_fwd_mg_quadratic`, :func:`kata_decode_step_mg` -- KATA-Mg, with
  several PSD factors per head (score sum_j (q^j . k^j)^2), the forward in
  the [B,H,T,d] or [B,T,H,d] layout;
* :func:`parallel_kata_attn` -- the pages' call shape, [B,T,H,D] in and out;
* :func:`kata_fwd_quadratic_train`, :func:`kata_bwd_quadratic` -- the forward
  that also returns the denominators, and the backward pass;
  :func:`kata_attention` wraps them as an autograd function;
  :func:`kata_fwd_chunked_train`, :func:`kata_bwd_chunked`,
  :func:`kata_attention_chunked` -- the same on the O(T) chunked path;
* :func:`kata_fwd_mg_chunked` -- KATA-Mg on the exact O(T) chunked path;
* :func:`kata_fwd_sg_quadratic`, :func:`kata_fwd_sg_chunked`,
  :func:`kata_decode_step_sg` -- KATA-Sigma-g, summed PSD factors (weight
  sum_{j,l} (q^j . k^l)^2): flash-style and chunked forward, decode;
  :func:`kata_fwd_sg_quadratic_train`, :func:`kata_bwd_sg_quadratic`,
  :func:`kata_attention_sg` -- its training forward and backward;
* :func:`kata_fwd_mg_quadratic_train`, :func:`kata_bwd_mg_quadratic`,
  :func:`kata_attention_mg` -- the same for KATA-Mg ([B,H,T,d]);
* :func:`kata_fwd_linear_chunked`, :func:`kata_fwd_linear_chunked_sequential`
  -- first-order (psi(u) = u) attention, chunked with the associative scan
  and its matched sequential baseline.
"""
from ._abi import (KataError, kata_abi_version, kata_decode_step, kata_fwd_chunked,  # noqa: F401
                   kata_fwd_chunked_noalloc, kata_fwd_chunked_sequential, kata_fwd_chunked_workspace_size,
                   kata_fwd_quadratic, kata_fwd_mg_quadratic, kata_decode_step_mg, parallel_kata_attn,
                   kata_fwd_quadratic_train, kata_bwd_quadratic, kata_attention, KataAttention,
                   kata_fwd_chunked_train, kata_bwd_chunked, kata_attention_chunked, KataAttentionChunked,
                   kata_fwd_mg_quadratic_train, kata_bwd_mg_quadratic, kata_attention_mg, KataAttentionMg,
                   kata_fwd_sg_quadratic, kata_decode_step_sg, kata_fwd_sg_chunked,
                   kata_fwd_sg_chunked_workspace_size, kata_fwd_sg_quadratic_train, kata_bwd_sg_quadratic,
                   kata_attention_sg, KataAttentionSg, kata_fwd_mg_chunked, kata_fwd_mg_chunked_workspace_size,
                   kata_fwd_linear_chunked, kata_fwd_linear_chunked_sequential,
                   kata_fwd_linear_chunked_workspace_size,
                   kata_get_status, kata_set_wait_limit, lib, status_string)
