"""fp64 CPU oracle for the Multi-Latent Attention forward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import or run it.  It shares no
code with the CUDA library (no kernels, headers, tables or helpers); the only
thing both sides use is the seeded input package ``mla_inputs``.

Functions and what pins them (tests/test_oracle_pins.py):

* ``yarn_get_mscale`` / ``softmax_scale`` -- closed form, golden values.
* ``rope_frequencies`` / ``rope_tables`` -- RoPE identities (norm
  preservation, rotate_half^2 = -I, relative-position property, factor 1
  reduces YaRN to plain RoPE, ramp end points).  The YaRN ramp's integer
  boundary choice (floor/ceil of the correction dimensions) is a reading of
  pages that give only the parameter names: **parity unpinned** for that
  choice beyond the end-point pins.
* ``prefill`` -- brute-force loop MHA (explicit per-head K, V zero-padded to
  the query head dim and trimmed), causality, softmax rows summing to 1,
  T=1 and equal-key special cases.
* ``decode_absorbed`` / ``decode_unabsorbed`` -- agree with each other and
  with the last row of a prefill.
* ``prefill_chunked`` -- equals the last rows of a full prefill whose first
  positions produced the cache; reduces to ``prefill`` with no history.
* ``prefill_varlen`` -- equals separate ``prefill`` calls on each packed
  sequence (block-diagonal mask vs separate problems); one sequence reduces
  to ``prefill``; one-token sequences return their own value row.
"""
from .mla_oracle import (yarn_get_mscale, softmax_scale, rope_frequencies,
                         rope_tables, rms_norm, rotate_half, apply_rope,
                         prefill, prefill_chunked, prefill_varlen,
                         decode_absorbed,
                         decode_unabsorbed, max_rel_err)

__all__ = ["yarn_get_mscale", "softmax_scale", "rope_frequencies",
           "rope_tables", "rms_norm", "rotate_half", "apply_rope", "prefill",
           "prefill_chunked", "prefill_varlen",
           "decode_absorbed", "decode_unabsorbed", "max_rel_err"]
