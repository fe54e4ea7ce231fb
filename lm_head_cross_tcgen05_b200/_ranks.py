"""The exchange steps the multi-rank drivers share. Each one only moves data between the ranks
of a torch.distributed group; the additions that combine the moved values run in the library's
kernels (through the driver's ``ops``), always in ascending rank order, so no floating-point
value is reduced inside a collective and the results are bitwise reproducible for a given
rank count."""
from __future__ import annotations

import torch
import torch.distributed as dist


def row_slices(N: int, R: int):
    """The rows [a, b) whose sum rank j computes: N split as evenly as possible, in order."""
    base, extra = divmod(N, R)
    out, a = [], 0
    for j in range(R):
        b = a + base + (1 if j < extra else 0)
        out.append((a, b))
        a = b
    return out


class RankGroup:
    """The ranks of ``group`` (or the default group). Without an initialised process group it
    runs as the only rank (R = 1, no collective)."""

    def __init__(self, group=None, ops=None):
        self.group = group
        self.distributed = dist.is_available() and dist.is_initialized()
        self.R = dist.get_world_size(group) if self.distributed else 1
        self.rank = dist.get_rank(group) if self.distributed else 0
        self.ops = ops

    def _gather(self, rec):
        """[N, w] records of this rank -> [R, N, w] of all ranks in rank order."""
        N, w = rec.shape
        if self.R == 1:
            return rec.view(1, N, w)
        every = torch.empty(self.R * N * w, dtype=rec.dtype, device=rec.device)
        dist.all_gather_into_tensor(every, rec.reshape(-1).contiguous(), group=self.group)
        return every.view(self.R, N, w)

    def _count_sum(self, n):
        """The sum over the ranks of an integer count tensor (exact in any order)."""
        if self.R == 1:
            return n
        total = n.clone()
        dist.all_reduce(total, op=dist.ReduceOp.SUM, group=self.group)
        return total

    def _sum_rows(self, part: torch.Tensor) -> torch.Tensor:
        """sum over ranks of part [N, d], added in ascending rank order, on every rank: an
        all-to-all hands rank j slice j of every rank's part, ``ops.reduce_rows`` adds them,
        and an all-gather returns the summed slices."""
        N, d = part.shape
        if self.R == 1:
            return self.ops.reduce_rows(part.view(1, N, d))
        sl = row_slices(N, self.R)
        sizes = [b - a for a, b in sl]
        mine = sizes[self.rank]
        recv = torch.empty(self.R * mine, d, dtype=part.dtype, device=part.device)
        dist.all_to_all_single(recv, part.contiguous(), output_split_sizes=[mine] * self.R,
                               input_split_sizes=sizes, group=self.group)
        red = self.ops.reduce_rows(recv.view(self.R, mine, d))
        top = max(sizes)
        if top == 0:
            return red
        if mine == top:
            pad = red
        else:  # slices differ by one row at most: gather equal blocks, drop the padding
            pad = torch.zeros(top, d, dtype=red.dtype, device=red.device)
            pad[:mine] = red
        every = torch.empty(self.R * top, d, dtype=red.dtype, device=red.device)
        dist.all_gather_into_tensor(every, pad.contiguous(), group=self.group)
        if all(n == top for n in sizes):
            return every
        return torch.cat([every[j * top: j * top + sizes[j]] for j in range(self.R)])
