"""Ring attention on B200: exact softmax attention folded chunk by chunk, forward and backward.

Public calls (thin wrappers over the C-ABI library ``libra.so``; every step of the
path runs in its CUDA kernels, there is no CPU fallback):

* ``partial(q, k, v, ...)``        one query block against one KV chunk -> (O_partial, lse)
* ``merge(o_parts, lse_parts)``    lse-weighted combination of partial states
* ``ring_forward(q, k, v, ...)``   the full ordered ring over virtual positions -> (O, lse)
* ``backward_delta(o, d_o)``       the row term D = rowsum(dO * O)
* ``partial_backward(...)``        one query block against one KV chunk, added into dQ/dK/dV
* ``ring_backward(...)``           gradients of ``ring_forward`` (``ring_backward_noalloc``:
                                   the same with the library's static scratch)

Across GPUs (one process per GPU, ``torch.distributed``): ``ring_dist`` (K||V sent around the
ring), ``peer_ring`` (K/V read from the owner's memory through CUDA IPC) and ``usp`` (Ulysses
all-to-all inside a group, the ring across groups).

The binding module loads the shared library on first use and raises if it is missing.
``sequence_softmax_b200.inputs`` (seeded inputs, workload shapes) imports without it.
"""

__all__ = ["partial", "partial_fold", "key_norm_max", "merge", "ring_forward", "backward_delta", "partial_backward",
           "ring_backward", "ring_backward_noalloc", "ring_backward_workspace_bytes", "status_string",
           "get_device_error", "selftest_wait_timeout", "library_path", "RaError"]


def __getattr__(name):
    if name in __all__:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
