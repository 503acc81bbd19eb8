"""The usage example: the forward on the GDN-2 workload's shapes, then a backward through
the autograd wrapper, as a function the GPU test runs."""


def run():
    import torch
    from matrix_memory_rnn_b200 import gdr
    from matrix_memory_rnn_b200.autograd import gdr_chunked

    B, T, H, d = 4, 4096, 16, 128
    bf = dict(dtype=torch.bfloat16, device="cuda")
    q, k, v = (torch.randn(B, T, H, d, **bf) for _ in range(3))
    k = torch.nn.functional.normalize(k.float(), dim=-1).to(torch.bfloat16)
    log_w = -0.05 * torch.rand(B, T, H, d, device="cuda")           # log of the decay, <= 0
    b = torch.sigmoid(torch.randn(B, T, H, d, **bf))                  # GDN-2 erase gate
    o, S_T = gdr.gdr_forward_chunked("gdn2", q, k, v, log_w, b)       # o [B, T, H, d] fp32

    q.requires_grad_(True)
    o, S_T = gdr_chunked("gdn2", q, k, v, log_w, b)
    o.sum().backward()                                                # q.grad via gdr_backward_chunked
    return dict(o=o, S_T=S_T, q=q)
