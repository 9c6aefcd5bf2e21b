"""Data parallelism over tokens for the fused LoRA linear layer.

Every rank holds the frozen weight W and the adapters A, B and runs the layer on its
own rows of x and dY.  h and dX depend only on a rank's own rows, so they stay local.
dA = s * sum_m g[m]^T x[m] and dB = s * sum_m dY[m]^T xa[m] are sums over tokens, so
the gradient of the whole batch is the sum of the ranks' gradients: the one exchange
per layer is a sum all-reduce of dA and dB.  They are written by the backward
straight into one packed fp32 buffer [dA | dB] (r*d_in + d_out*r floats), so the
all-reduce is a single call with no packing copy.  Page "ms-swift高效微调组合：LoRA+
UnSloth提速实践", section 1.1, names the multi-GPU all-reduce of the adapter gradients
as a cost of plain LoRA training; page "UnSloth加速库集成：编译级优化带来的性能飞跃",
sections 核心技术一 (one gradient sync for A and B) and 技术二 (packed A/B layout),
describes the remedy this module follows.  Only the adapters are exchanged: W is
frozen and has no gradient.

The sum is what the layer's definition gives (dA, dB of L = sum over all tokens);
averaging over ranks, if wanted, belongs in the loss scale.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def token_shard(M: int, world: int, rank: int) -> tuple[int, int]:
    """(first row, row count) of rank's share of M tokens: contiguous, sizes differ by
    at most one, the first M % world ranks take the extra row."""
    if world < 1 or not 0 <= rank < world or M < 0:
        raise ValueError(f"bad shard request M={M} world={world} rank={rank}")
    base, extra = divmod(M, world)
    return rank * base + min(rank, extra), base + (1 if rank < extra else 0)


class PackedGrads:
    """fp32 [dA | dB] in one contiguous buffer.

    ``dA`` ([r, d_in]) and ``dB`` ([d_out, r]) are row-major views into it, in the
    layouts lora_linear_bwd writes, so the backward fills the buffer directly.
    """

    def __init__(self, r: int, d_in: int, d_out: int, device=None):
        self.r, self.d_in, self.d_out = r, d_in, d_out
        self.buf = torch.empty(r * d_in + d_out * r, dtype=torch.float32, device=device)
        self.dA = self.buf[: r * d_in].view(r, d_in)
        self.dB = self.buf[r * d_in:].view(d_out, r)

    def zero_(self) -> "PackedGrads":
        """For a rank with no tokens this step: it still takes part in the all-reduce."""
        self.buf.zero_()
        return self

    def all_reduce(self, group=None, async_op: bool = False):
        """Sum [dA | dB] over the ranks of ``group`` in place (one collective)."""
        return dist.all_reduce(self.buf, op=dist.ReduceOp.SUM, group=group, async_op=async_op)
