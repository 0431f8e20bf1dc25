"""B200-native MLA decoding over a paged latent KV cache.

The compute path is libmla_b200.so (hand-written sm_100a CUDA: TMA, tcgen05
UMMA with TMEM accumulators) behind the C ABI of include/mla.h; this package
re-exports its thin ctypes binding.  ``workloads`` holds the seeded synthetic
input generators.
"""

_BINDING_NAMES = (
    "mla_num_sm_parts", "mla_get_metadata", "mla_get_metadata_host", "mla_workspace_size",
    "mla_sparse_workspace_size", "mla_decode_fwd", "mla_fused_norm_rope_attn_rope_cast",
    "mla_sparse_decode", "device_status", "MLAError", "lib",
)


def __getattr__(name):
    # Load the CUDA binding lazily so that importing the input generators
    # does not require the shared library.
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
