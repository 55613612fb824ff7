"""Shared plumbing of the GPU parity tests: run a workload step through the
C ABI (via the binding) and through the CPU oracle on the same input bits.

Tolerance: the attention target is a max absolute error of 2e-3 between the
FP32 GPU output and the FP64 oracle on BF16 inputs.  Append and page
indexing must match bit for bit.
"""
import numpy as np
import torch

import oracle
from paged_attention_decode_pkv_b200 import pkv
from paged_attention_decode_pkv_b200 import workloads as W

ATOL = 2e-3
KERNELS = [pkv.KERNEL_SIMT, pkv.KERNEL_MMA]


def bits(t):
    return W.bits(t)


def to_dev(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def u16_to_bf16(a, device="cuda"):
    return to_dev(np.ascontiguousarray(a, np.uint16).view(np.int16), device).view(torch.bfloat16)


class GpuCase:
    """A small case (tests.cases.make_case dict) loaded on the GPU."""

    def __init__(self, case, device="cuda"):
        self.case = case
        self.pool_t = u16_to_bf16(case["pool"], device)
        self.pool = pkv.Pool(case["pool"].shape[0], storage=self.pool_t)
        self.bt = to_dev(case["bt"], device)
        self.sl = to_dev(case["seq_lens"], device)
        self.q = u16_to_bf16(case["q"], device)

    def decode(self, layer=0, scale=0.125, **kw):
        out = pkv.decode(self.q, self.pool, self.bt, self.sl, layer, scale, **kw)
        torch.cuda.synchronize()
        return out.cpu().numpy().astype(np.float64)

    def oracle(self, layer=0, scale=0.125):
        c = self.case
        return oracle.decode(c["q"], c["pool"], c["bt"], c["seq_lens"], layer, scale)


def max_err(got, want):
    return float(np.max(np.abs(got - want))) if got.size else 0.0
