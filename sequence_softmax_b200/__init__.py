"""Ring attention forward on one B200: exact softmax attention folded chunk by chunk.

Public calls (thin wrappers over the C-ABI library ``libra.so``; every step of the
path runs in its CUDA kernels, there is no CPU fallback):

* ``partial(q, k, v, ...)``      one query block against one KV chunk -> (O_partial, lse)
* ``merge(o_parts, lse_parts)``  lse-weighted combination of partial states
* ``ring_forward(q, k, v, ...)`` the full ordered ring over virtual positions -> (O, lse)

The binding module loads the shared library on first use and raises if it is missing.
``sequence_softmax_b200.inputs`` (seeded inputs, workload shapes) imports without it.
"""

__all__ = ["partial", "merge", "ring_forward", "status_string", "get_device_error",
           "selftest_wait_timeout", "library_path", "RaError"]


def __getattr__(name):
    if name in __all__:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
