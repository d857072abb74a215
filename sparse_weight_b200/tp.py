"""Row-sharded (tensor-parallel) decode of a packed hybrid matrix.

Each rank of a process group holds a contiguous range of tile-row bands
(hyb_shard_bands: balanced by packed bytes), applies it to the full input with
the library's product, and the ranks' rows are gathered into the full output
with one all-gather (NCCL over NVLink on GPUs, gloo on CPU).  This module is
plumbing around the C ABI: shard views, padding to the largest shard, the
collective and the reassembly; every product runs in the library's kernels.
"""
from typing import Callable, Optional

import torch
import torch.distributed as dist

from . import hyb


class RowShard:
    """Rank `rank`'s share of A for a row-sharded product over `world` ranks."""

    def __init__(self, A: hyb.Packed, rank: int, world: int, plan: bool = True):
        self.n, self.k, self.b1 = A.n, A.k, A.b1
        self.rank, self.world = rank, world
        self.bands = [hyb.shard_bands(A.n, A.k, A.b1, A.b2, A.tile_map, world, r)
                      for r in range(world)]
        self.rows = [(b0 * A.b1, b1 * A.b1) for b0, b1 in self.bands]
        self.max_rows = max(hi - lo for lo, hi in self.rows)
        self.local = hyb.shard(A, rank, world, plan=plan)
        self._bufs = {}  # (batch, device) -> (shard output, gather buffer, Y)

    def _buffers(self, batch, device):
        key = (batch, str(device))
        if key not in self._bufs:
            self._bufs[key] = (
                torch.zeros(batch, self.max_rows, dtype=torch.float32, device=device),
                torch.empty(self.world * batch, self.max_rows, dtype=torch.float32, device=device),
                torch.empty(batch, self.n, dtype=torch.float32, device=device))
        return self._bufs[key]

    def apply(self, X: torch.Tensor, group=None,
              product: Optional[Callable[[hyb.Packed, torch.Tensor, Optional[torch.Tensor]],
                                         torch.Tensor]] = None,
              **kwargs) -> torch.Tensor:
        """Y[batch][n] = W_hat X on every rank: this rank's rows by
        `product(shard, X, out)` (default hyb.spmm_skinny; `out` is the padded
        buffer when the shard fills it, else None), then one all-gather of the
        padded shard outputs ([world][batch][max_rows] fp32) and the
        reassembly."""
        if product is None:
            def product(S, x, out):
                return hyb.spmm_skinny(S, x, Y=out, **kwargs)
        Xb = X if X.dim() == 2 else X.view(1, -1)
        batch = Xb.shape[0]
        # (buffers reused across calls; the returned Y is overwritten by the
        # next call with the same batch)
        buf, flat, Y = self._buffers(batch, Xb.device)
        if self.local is not None:
            lo, hi = self.rows[self.rank]
            if hi - lo == self.max_rows:
                product(self.local, Xb, buf)
            else:
                buf[:, :hi - lo] = product(self.local, Xb, None)
        # the ranks' buffers concatenated along dim 0 (the form both NCCL and
        # gloo accept), then seen as [world][batch][max_rows]
        if self.world > 1:
            dist.all_gather_into_tensor(flat, buf, group=group)
        else:
            flat.copy_(buf)
        gathered = flat.view(self.world, batch, self.max_rows)
        for r, (lo, hi) in enumerate(self.rows):
            Y[:, lo:hi] = gathered[r, :, :hi - lo]
        return Y
