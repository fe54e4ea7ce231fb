"""The exchange steps the multi-rank classes (VocabParallelCE, VocabParallelSupport,
DataParallelCE) share. Each one only moves data between the ranks of a torch.distributed
group; the additions that combine the moved values run in the library's kernels (through the
class's ``ops``), always in ascending rank order, so no floating-point value is reduced inside
a collective and the results are bitwise reproducible for a given rank count."""
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
        self._sym = None

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

    # ------------------------------------------------------------- peer-memory exchange
    # Waits of the peer-memory barrier give up after this long (the library's bounded wait):
    # a rank that never arrives leaves the others an error to read, not a GPU that spins.
    barrier_timeout_ms = 4000

    def _symmetric(self, rows, d, device):
        """For a sum over the ranks of [rows, d] fp32 parts, in symmetric memory (peer-mapped
        over NVLink): the receive buffer of this rank ([R][rows_j][d] fp32 within
        R * max_j rows_j * d) and the full bf16 [rows, d] output of every rank, with the
        device tables of the R ranks' addresses of both; and the signal arrays of the
        library's barrier (R uint32 words per rank, zeroed on every rank before first use)."""
        if self._sym is not None and self._sym["key"] == (rows, d):
            return self._sym
        import torch.distributed._symmetric_memory as symm_mem
        group = self.group if self.group is not None else dist.group.WORLD
        sizes = [b - a for a, b in row_slices(rows, self.R)]
        n_recv = self.R * max(sizes) * d
        recv = symm_mem.empty(n_recv, dtype=torch.float32, device=device)
        recv_h = symm_mem.rendezvous(recv, group)
        out = symm_mem.empty(rows * d, dtype=torch.bfloat16, device=device)
        out_h = symm_mem.rendezvous(out, group)
        sig = symm_mem.empty(self.R, dtype=torch.int32, device=device)
        sig_h = symm_mem.rendezvous(sig, group)
        sig.zero_()
        torch.cuda.synchronize(device)
        self._host_barrier(device)           # every rank's signal words are zero

        def table(h, n, dtype):
            return torch.tensor([h.get_buffer(r, (n,), dtype).data_ptr() for r in range(self.R)],
                                dtype=torch.int64, device=device)
        self._sym = dict(key=(rows, d), sizes=sizes, recv=recv, recv_h=recv_h, out=out,
                         out_h=out_h, recv_tab=table(recv_h, n_recv, torch.float32),
                         out_tab=table(out_h, rows * d, torch.bfloat16), sig=sig, sig_h=sig_h,
                         sig_tab=table(sig_h, self.R, torch.int32), epoch=0,
                         err=torch.zeros(256, dtype=torch.uint8, device=device))
        return self._sym

    def _host_barrier(self, device):
        """All ranks reach this point (a one-element all-reduce, waited for on the host)."""
        t = torch.zeros(1, dtype=torch.int32, device=device)
        dist.all_reduce(t, group=self.group)
        torch.cuda.synchronize(device)

    def _barrier(self, sym):
        """The library's peer-memory barrier on the current stream (bounded wait)."""
        from . import lmh_peer_barrier
        sym["epoch"] = (sym["epoch"] + 1) & 0xFFFFFFFF or 1
        lmh_peer_barrier(sym["err"], sym["sig_tab"], self.R, self.rank, sym["epoch"],
                         self.barrier_timeout_ms)

    def check_exchange(self):
        """Raise if a peer-memory barrier of this rank gave up waiting. Synchronises the
        current stream (it reads the barriers' device error word)."""
        if self._sym is None:
            return
        from . import DEVERR_TIMEOUT, lmh_read_errors
        bits = lmh_read_errors(self._sym["err"])
        if bits:
            self._sym["err"].zero_()
            raise RuntimeError(
                "peer-memory exchange: a barrier timed out waiting for another rank"
                if bits & DEVERR_TIMEOUT else f"peer-memory exchange: device error {bits:#x}")

    def _open_p2p(self, rows, d, device):
        """The symmetric buffers, after checking the previous exchange and a barrier that
        lets every rank reuse its receive buffer (no rank still reads its last contents)."""
        self.check_exchange()
        sym = self._symmetric(rows, d, device)
        self._barrier(sym)
        return sym

    def _reduce_p2p(self, sym):
        """After every rank's rows landed: reduce this rank's slice into every rank's output."""
        sizes = sym["sizes"]
        mine, start = sizes[self.rank], sum(sizes[:self.rank])
        d = sym["key"][1]
        self._barrier(sym)                    # every rank's rows are in the receive buffers
        parts = sym["recv"][: self.R * mine * d].view(self.R, mine, d)
        self.ops.reduce_rows_to(parts, sym["out_tab"], self.R, start)
        self._barrier(sym)                    # every rank's slice is in every output
        return sym["out"].view(-1, d).clone()
