"""Usage example of the la2 binding (the one README.md shows): forward,
backward, decay gradient, recurrent decode and a packed batch on a B200.

Run as a script, or call main() (the GPU test suite does) to get the
outputs by name."""
import torch

import causal_linear_attention_fwd_b200 as la2


def main():
    B, H, L, d = 4, 16, 2048, 128
    q, k, v, dO = (torch.randn(B, H, L, d, device="cuda", dtype=torch.bfloat16) for _ in range(4))
    lam = torch.tensor([1 - 2 ** -(5 + 8 * h / H) for h in range(H)], device="cuda")  # decay per head

    o, kv = la2.forward(q, k, v, lam, want_state=True)             # O = (QK^T (.) M) V, final state
    dq, dk, dv = la2.backward(q, k, v, lam, dO)                    # gradients of sum(O * dO)
    dlam = la2.dlambda(q, k, v, lam, dO)                           # gradient w.r.t. each head's decay

    # recurrent decode from the state the forward left: one token, or T tokens per call
    q1, k1, v1 = (torch.randn(B, H, d, device="cuda", dtype=torch.bfloat16) for _ in range(3))
    o1 = la2.decode_step(q1, k1, v1, lam, kv)                      # kv updated in place
    qT, kT, vT = (torch.randn(B, H, 32, d, device="cuda", dtype=torch.bfloat16) for _ in range(3))
    oT = la2.decode_tokens(qT, kT, vT, lam, kv)                    # 32 tokens per request at once

    # packed variable-length batch: documents back to back in [H, T, d], int64 offsets
    cu = torch.tensor([0, 300, 1000, 2048], dtype=torch.int64, device="cuda")  # 3 documents
    qp, kp, vp = (t[0].contiguous() for t in (q, k, v))           # [H, 2048, d]
    op = la2.forward_varlen(qp, kp, vp, lam, cu)
    return dict(o=o, dq=dq, dk=dk, dv=dv, dlam=dlam, o1=o1, oT=oT, op=op)


if __name__ == "__main__":
    out = main()
    torch.cuda.synchronize()
    print({name: tuple(t.shape) for name, t in out.items()})
