"""Representative calls of every entry point for the checked-build test: ragged tiles, all
three layouts, causal and not, fp32 and bf16, both head dimensions, token offsets and
strides, empty partial states. run_cases() returns the outputs by name; run as a script it
writes them to an .npz file and fails if the device error word is set after any call."""

from __future__ import annotations

import sys

import numpy as np
import torch


def run_cases():
    from sequence_softmax_b200 import binding
    from sequence_softmax_b200.inputs import make_qkv

    out = {}

    def record(name, tensors):
        assert binding.get_device_error() == binding.RA_OK, name
        out[name] = [t.float().cpu().numpy() for t in tensors]

    for (dt, N, d, P, layout, causal) in [(torch.bfloat16, 1000, 128, 4, "zigzag", True),
                                          (torch.bfloat16, 1000, 64, 4, "striped", True),
                                          (torch.bfloat16, 768, 128, 3, "contiguous", False),
                                          (torch.float32, 96, 128, 4, "striped", True)]:
        q, k, v = make_qkv(1, 2, N, d, dt, seed=N + d, device="cuda")
        do = make_qkv(1, 2, N, d, dt, seed=N + d + 1, device="cuda")[0]
        o, lse = binding.ring_forward(q, k, v, P, causal, layout)
        record(f"fwd-{layout}-{N}-{d}-{dt}", (o, lse))
        grads = binding.ring_backward(q, k, v, o, do, lse, P, causal, layout)
        record(f"bwd-{layout}-{N}-{d}-{dt}", grads)
    q, _, _ = make_qkv(1, 2, 300, 128, torch.bfloat16, seed=3, device="cuda")
    _, k, v = make_qkv(1, 2, 333, 128, torch.bfloat16, seed=4, device="cuda")
    o_p, l_p = binding.partial(q, k, v, causal=True, q_tok0=5, q_tok_stride=16, k_tok0=2, k_tok_stride=16)
    record("partial-striped", (o_p, l_p))
    o_e, l_e = binding.partial(q, k, v, causal=True, q_tok0=0, k_tok0=10 ** 6)  # every row empty
    record("partial-empty", (o_e, l_e))
    m_o, m_l = binding.merge(torch.stack([o_p, o_e, o_p]), torch.stack([l_p, l_e, l_p]), out_dtype=torch.bfloat16)
    record("merge-with-empty", (m_o, m_l))
    do = make_qkv(1, 2, 300, 128, torch.bfloat16, seed=5, device="cuda")[0]
    delta = binding.backward_delta(o_p.to(torch.bfloat16), do)
    acc = [torch.zeros(1, 2, 300, 128, device="cuda"), torch.zeros(1, 2, 333, 128, device="cuda"),
           torch.zeros(1, 2, 333, 128, device="cuda")]
    binding.partial_backward(q, k, v, do, l_p, delta, *acc, causal=True, q_tok0=5, q_tok_stride=16, k_tok0=2,
                             k_tok_stride=16)
    record("partial-backward-striped", acc + [delta])
    return out


if __name__ == "__main__":
    res = run_cases()
    np.savez(sys.argv[1], **{f"{k}|{i}": a for k, v in res.items() for i, a in enumerate(v)})
    print("checked cases ok:", len(res))
