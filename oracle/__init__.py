"""fp64 CPU oracle for MLA latent-KV decode and prefill.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / reference leg of ``bench.py`` may import this
package.  The CUDA library never calls it and shares no code with it.

The oracle computes Multi-head Latent Attention in its plain, unabsorbed
(decompressed MHA) form, following the sources cited in ``mla_oracle``:
per head it rebuilds K = [c_KV W_UK | RoPE(k_pe)] and V = c_KV W_UV from the
cached latent and runs naive softmax attention in float64.

Pin status: every public function is pinned by ``tests/test_oracle_pins.py``
(worked example, closed forms, invariants, brute force, library routines).
Nothing here is "parity unpinned".
"""
from .mla_oracle import (  # noqa: F401
    rope_frequencies, rope_rotate, rms_norm, append_latent, gather_rows,
    decompress_head, attend, decode, decode_one, decode_sparse, prefill, query_from_hidden,
    output_projection, kv_cache_bytes_mha,
    latent_elems_per_token,
)
