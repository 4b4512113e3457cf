"""fp64 CPU oracle for the ReplaySSM decode path.

THIS IS TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import it.  The product (the CUDA
library under ``hybrid_ssm_decode_replayssm_b200``) never imports, links or
calls anything here, and nothing here imports the product.  The only code the
two sides share is ``seeded_inputs``, which draws inputs and holds none of the
method's arithmetic.

What it computes and why that is the right answer
-------------------------------------------------
ReplaySSM changes how a layer's state is *stored* (a checkpoint plus a buffer
of recent inputs, replayed on every read), not what a decode step outputs.
The pages say the change "separates output computation from state updates"
and that a replayed state should equal the stored one; so the oracle for every
ReplaySSM output and checkpoint is the plain token-by-token recurrence of the
layer, in fp64 (``mamba2``, ``gdn``).  The replay form itself is restated in
fp64 in ``replay`` so that its algebra can be checked against the recurrence.

Citation legend (all three pages carry the title "ReplaySSM: Rethinking State
Storage for Faster Hybrid-Model Decoding"):

* [teaser]        babnews.org RSS teaser (names Mamba-2, GDN and KDA layers).
* [summary ¶n]    deskofai.com news summary, paragraph n.  ¶2: checkpoint plus
                  buffer of recent inputs, output separated from state update;
                  ¶3: cache the inputs, flush when the buffer fills, append
                  drafts, roll back by moving a pointer; ¶4: high-precision
                  checkpoint for the recurrence plus a low-precision (NVFP4)
                  read copy; ¶6: window L = 16.
* [guide §name]   nexus-ai-blog.com how-to article, section "name".

Modules and what pins each one (tests marked ``not gpu``):

* ``mamba2``      conventional Mamba-2 recurrence.  Pinned by a brute-force
                  unrolled closed form (tiny P, N, T), the scalar geometric
                  series, and the A = 0, dt = 1 reduction to causal linear
                  attention (cumulative sum of outer products).
* ``gdn``         conventional gated delta rule.  Pinned by the explicit
                  product-of-transitions closed form (d <= 4), beta = 0 pure
                  decay, and exact key/value memorisation with orthonormal keys.
* ``replay``      replay form (Mamba-2 SSD window sum; GDN WY/UT forward
                  substitution) with flush.  Pinned against ``mamba2``/``gdn``
                  for L in {1, 2, 3, 4, 8, 16, 32} (agreement to 1e-12).
* ``codecs``      OCP FP8 E4M3 and FP4 E2M1 encoders/decoders and the two
                  read-copy quantisers.  Pinned by the spec's code tables
                  (tests/golden), torch's float8_e4m3fn cast, and midpoint
                  tie cases.
* ``bookkeeping`` window pointer rules (start, len, pending, flushes).  Pinned
                  by an explicit list-of-tokens model and a hand-traced fixture.
* ``speculative`` verify/rollback reference: k drafts run conventionally from
                  the committed state, committed state advanced by the accepted
                  prefix.  Pinned by the rollback invariant (equal to decoding
                  only the accepted tokens from scratch).
* ``quantized_state`` the baseline a read copy replaces: the conventional
                  update on a state stored in FP8/NVFP4 and rounded again every
                  token [summary ¶4].  Pinned by exactly representable states
                  being fixed points of a do-nothing token, by the output being
                  the one of the state before rounding, and by its drift over
                  many tokens exceeding one rounding of the exact state.

* ``kda``         Kimi Delta Attention (reading: the gated delta rule with a
                  per-key-channel gate) and its replay form.  Pinned by the
                  gated delta rule it reduces to with equal channel gates, the
                  explicit product of transitions (d <= 4), beta = 0 channel
                  decay, orthonormal-key memorisation, and replay equal to the
                  recurrence for L in {1, 2, 3, 4, 8, 16, 32}.
* ``branch``      branch/fork (rows continue from other rows' states) and
                  restore-to-position [guide §"The State-Storage Bottleneck in
                  Branching Workloads", §"What a Replay-First Design
                  Implies"].  Pinned by recomputing every row's state from its
                  own token lineage (a list of tokens copied at each branch),
                  and by the identity / single-parent / full-window special
                  cases.

No function here is "parity unpinned".
"""
from . import bookkeeping, branch, codecs, gdn, kda, mamba2, quantized_state, replay, speculative  # noqa: F401
