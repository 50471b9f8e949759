"""Branch-parallel MLRA decode: the branches spread over devices, one or more per device.

"Multi-Head Low-Rank Attention" (yunpan.plus page), sections 3.2 and 4: MLRA-B splits the latent
state into B blocks c_1 .. c_B whose attentions are independent (each branch has its own softmax)
and are summed only after the value up-projection.  With B devices of tensor parallelism, device b
keeps only its block c_b (d_c / B columns) and the RoPE key k^R shared by all branches, so that per
cached token it reads d_R + d_c / B elements instead of the d_R + d_c of MLA; it runs steps 2
and 3 for its branch alone, and one all-reduce (sum) after step 3 gives every device the layer's
attention output:

    y[s, h] = sum_b  W^UV_{h,b} (gamma * o_b[s, h])        o_b: branch b's attention output

Device b's arrays are the b-th column blocks of the full ones (cut once, at load), and its decode is
the single-branch decode (num_branches = 1) with the full layer's softmax scale and branch scale
gamma = 1 / B.  The all-reduce goes through torch.distributed (NCCL between GPUs).

With fewer devices than branches (G devices, G dividing B), device g keeps the g-th of G equal
column blocks, i.e. B / G adjacent branches, and runs the B / G-branch decode on it (still with
gamma = 1 / B); the branches' softmaxes stay independent, so the sum over devices is unchanged.
The helpers below cut G equal blocks whatever G is.
"""
from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist

from . import mlra

__all__ = ["branch_block", "shard_latent", "shard_queries", "shard_wuv", "BranchShardStep"]


def branch_block(width: int, branch: int, num_branches: int) -> slice:
    """Columns of branch ``branch`` in a width-``width`` latent axis split into equal blocks."""
    if num_branches < 1 or width % num_branches or not 0 <= branch < num_branches:
        raise ValueError(f"branch {branch} of {num_branches} over width {width}")
    d = width // num_branches
    return slice(branch * d, (branch + 1) * d)


def shard_latent(c_kv: torch.Tensor, branch: int, num_branches: int) -> torch.Tensor:
    """Device ``branch``'s latent cache: its column block of c_kv [rows, d_c], contiguous."""
    return c_kv[:, branch_block(c_kv.shape[-1], branch, num_branches)].contiguous()


def shard_queries(q_lat: torch.Tensor, branch: int, num_branches: int) -> torch.Tensor:
    """Device ``branch``'s absorbed queries: its block of q_lat [N, H, d_c]."""
    return q_lat[..., branch_block(q_lat.shape[-1], branch, num_branches)].contiguous()


def shard_wuv(w_uv: torch.Tensor, branch: int, num_branches: int) -> torch.Tensor:
    """Device ``branch``'s value up-projections W^UV_{h,branch}: its column block of
    w_uv [H, d_head, d_c]."""
    return w_uv[..., branch_block(w_uv.shape[-1], branch, num_branches)].contiguous()


class BranchShardStep:
    """Steps 2 and 3 of this device's branches, then the sum over the branch devices.

    q_lat_b [N, H, d_c / G] and c_b [rows, d_c / G] are this device's blocks (``shard_queries``,
    ``shard_latent`` with G shards); q_rope, k_rope, seq_lens and page_table are the full
    (replicated) arrays; w_uv_b [H, d_head, d_c / G] bf16 is ``shard_wuv``'s block, packed here
    once.  ``num_branches`` is the layer's B and ``branches_per_device`` B / G (default 1: one
    branch per device).  ``group`` is the process group of the G devices (None: the default
    group); with ``reduce=False`` the call returns this device's share and leaves the sum to the
    caller.  The returned tensor is the step's output buffer, overwritten by the next call.
    """

    def __init__(self, q_lat_b, q_rope, c_b, k_rope, seq_lens, page_table, w_uv_b, *,
                 num_branches: int, softmax_scale: float, max_seq_len=None, page_size=0,
                 group: Optional[dist.ProcessGroup] = None, reduce: bool = True,
                 branches_per_device: int = 1):
        if branches_per_device < 1 or num_branches % branches_per_device:
            raise ValueError(f"{branches_per_device} branches per device of {num_branches}")
        self.num_branches = num_branches
        self.group = group
        self.reduce = reduce
        self.decoder = mlra.Decoder(q_lat_b, q_rope, c_b, k_rope, seq_lens, page_table,
                                    num_branches=branches_per_device, softmax_scale=softmax_scale,
                                    branch_scale=1.0 / num_branches, max_seq_len=max_seq_len,
                                    page_size=page_size)
        self.w_packed = mlra.pack_wuv(w_uv_b)
        N, H, _ = q_lat_b.shape
        self.y = torch.empty(N, H, w_uv_b.shape[1], dtype=torch.float32, device=q_lat_b.device)

    def local(self) -> torch.Tensor:
        """This device's share sum over its branches b of W^UV_{h,b} (gamma o_b) [N, H, d_head]
        (fp32)."""
        return mlra.project(self.decoder(), self.w_packed, self.y)

    def __call__(self) -> torch.Tensor:
        y = self.local()
        if self.reduce:
            dist.all_reduce(y, op=dist.ReduceOp.SUM, group=self.group)
        return y
