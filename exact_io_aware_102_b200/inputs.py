"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no attention arithmetic: it only draws the Q, K, V tensors
and the sampled query rows that both the CUDA path and the CPU oracle are fed.

Recipe (the pages give no data; their workload is image patches through a
model's input projection, which needs the model and images, so iid normals of
the same shapes stand in):

* one CPU ``torch.Generator`` seeded with ``seed``;
* Q, then K, then V drawn in that order as float32 N(0, 1) of shape
  [B, H, N, d] and rounded to bf16 (round to nearest even);
* the stability variant multiplies the bf16 Q by ``q_mult`` (4 is exact in bf16);
* sampled query rows per (b, h): rows 0 and N-1 plus rows drawn from
  ``torch.randperm(N)`` seeded with ``1000 + b*H + h``;
* the upstream gradient dO of the backward: float32 N(0, 1) [B, H, N, d]
  from its own generator seeded with ``seed``, rounded to bf16.
"""
import torch


def make_qkv(B, H, N, d, seed=0, q_mult=1.0):
    """Return bf16 CPU tensors (q, k, v), each [B, H, N, d] contiguous."""
    g = torch.Generator().manual_seed(int(seed))
    shape = (B, H, N, d)
    q = torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)
    if q_mult != 1.0:
        q = (q * q_mult).to(torch.bfloat16)
    return q, k, v


def make_dout(B, H, N, d, seed=1):
    """Return a bf16 CPU tensor dO [B, H, N, d] contiguous."""
    g = torch.Generator().manual_seed(int(seed))
    return torch.randn((B, H, N, d), generator=g, dtype=torch.float32).to(torch.bfloat16)


def sample_rows(B, H, N, count=256):
    """int64 tensor [B*H, R] of sorted distinct query rows per head (R = min(count, N))."""
    count = min(int(count), int(N))
    out = []
    for b in range(B):
        for h in range(H):
            if count >= N:
                out.append(torch.arange(N, dtype=torch.int64))
                continue
            g = torch.Generator().manual_seed(1000 + b * H + h)
            perm = torch.randperm(N, generator=g)
            chosen = [0, N - 1]
            for r in perm.tolist():
                if len(chosen) >= count:
                    break
                if r != 0 and r != N - 1:
                    chosen.append(r)
            out.append(torch.tensor(sorted(chosen), dtype=torch.int64))
    return torch.stack(out)
