"""N-sharded LLM.int8() forward: one block of output features per GPU.

The Hugging Face integration page serves the INT8 BLOOM-176B over several
GPUs ("Speed trade-offs", the table of BLOOM-176B runs).  The forward splits
along the output features N with no exchange inside the compute: every rank
holds rows [lo, hi) of CB, SCB and bias, reads the whole X, finds the same
outlier columns and row scales (they depend on X alone), and produces the
columns [lo, hi) of Y.  Two ways to assemble the full Y on every rank:

* ``mode="peer"`` -- the product kernel stores its column block into the
  output buffer of every rank directly (``int8_linear_forward_sharded`` with
  the peers' buffers as extra destinations; the buffers come from torch's
  symmetric memory, mapped into each GPU's address space).  The gather costs
  no extra pass over Y and overlaps the GEMM tile by tile; a stream-ordered
  barrier before (the previous Y may still be read) and after (every rank's
  stores have landed) brackets the call.
* ``mode="nccl"`` -- each rank computes its block into a local buffer and
  ``torch.distributed.all_gather`` moves the blocks; a concatenation along
  the columns assembles Y.  The plain collective, kept as the baseline.

Every step of the forward runs in libint8mp's kernels; this module only
splits the layer, sets up buffers and calls the collectives.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import native

SHARD_ALIGN = 16  # the library's rule for N (16-byte rows of CB and Y)


def shard_range(N: int, world: int, rank: int, align: int = SHARD_ALIGN) -> tuple[int, int]:
    """Contiguous output-feature block [lo, hi) of ``rank`` out of ``world``:
    multiples of ``align``, sizes differing by at most ``align``."""
    if N % align != 0:
        raise ValueError(f"N={N} is not a multiple of {align}")
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside [0, {world})")
    units = N // align
    if units < world:
        raise ValueError(f"N={N} gives fewer than {world} blocks of {align} features")
    base, rem = divmod(units, world)
    lo = (rank * base + min(rank, rem)) * align
    hi = lo + (base + (1 if rank < rem else 0)) * align
    return lo, hi


def shard_layer(CB: torch.Tensor, SCB: torch.Tensor, bias: torch.Tensor | None, world: int, rank: int):
    """This rank's rows of a quantised layer: (CB, SCB, bias, lo, hi)."""
    lo, hi = shard_range(CB.shape[0], world, rank)
    b = None if bias is None else bias[lo:hi].contiguous()
    return CB[lo:hi].contiguous(), SCB[lo:hi].contiguous(), b, lo, hi


def peer_destinations(local_ptr: int, buffer_ptrs: list[int], rank: int) -> list[int]:
    """Addresses of one symmetric output in every rank's buffer, this rank's
    first: the local tensor sits at the same offset in every rank's buffer."""
    off = local_ptr - int(buffer_ptrs[rank])
    if off < 0:
        raise ValueError("the tensor does not lie in this rank's symmetric buffer")
    return [local_ptr] + [int(p) + off for r, p in enumerate(buffer_ptrs) if r != rank]


def gather_columns(Y_shard: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather of the ranks' column blocks [T, n_r] into the full [T, N]
    (blocks in rank order; unequal widths allowed)."""
    world = dist.get_world_size(group)
    widths = [torch.zeros(1, dtype=torch.int64, device=Y_shard.device) for _ in range(world)]
    dist.all_gather(widths, torch.tensor([Y_shard.shape[1]], dtype=torch.int64, device=Y_shard.device), group=group)
    w = [int(x.item()) for x in widths]
    T, wmax = Y_shard.shape[0], max(w)
    if Y_shard.shape[1] == wmax:
        mine = Y_shard.contiguous()
    else:  # collectives move equal-sized blocks: pad to the widest shard
        mine = torch.zeros((T, wmax), dtype=Y_shard.dtype, device=Y_shard.device)
        mine[:, : Y_shard.shape[1]] = Y_shard
    parts = [torch.empty((T, wmax), dtype=Y_shard.dtype, device=Y_shard.device) for _ in range(world)]
    dist.all_gather(parts, mine, group=group)
    return torch.cat([p[:, :wr] for p, wr in zip(parts, w)], dim=1)


class NShardedLinear:
    """One rank's part of an N-sharded int8 linear layer.

    ``CB``, ``SCB``, ``bias``: the full quantised layer or already this rank's
    shard (``sharded=True``).  ``T_max``: the largest batch of tokens a
    forward will see (the output buffer is [T_max, N]).
    """

    def __init__(self, CB: torch.Tensor, SCB: torch.Tensor, bias: torch.Tensor | None, *, T_max: int,
                 dtype: torch.dtype = torch.float16, group=None, mode: str = "peer", sharded: bool = False,
                 N: int | None = None, path: int = native.PATH_AUTO):
        if mode not in ("peer", "nccl"):
            raise ValueError(f"mode {mode!r}")
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if sharded:
            if N is None:
                raise ValueError("N (the full output width) is required with sharded=True")
            self.N = N
            self.lo, self.hi = shard_range(N, self.world, self.rank)
            if CB.shape[0] != self.hi - self.lo:
                raise ValueError(f"shard has {CB.shape[0]} rows, expected {self.hi - self.lo}")
            self.CB, self.SCB, self.bias = CB, SCB, bias
        else:
            self.N = CB.shape[0]
            self.CB, self.SCB, self.bias, self.lo, self.hi = shard_layer(CB, SCB, bias, self.world, self.rank)
        self.K = self.CB.shape[1]
        self.mode, self.dtype, self.T_max, self.path = mode, dtype, T_max, path
        dev = self.CB.device
        n = self.hi - self.lo
        self.ws = native.new_workspace(T_max, self.K, n, dev)
        self.idx = torch.empty((self.K,), dtype=torch.int32, device=dev)
        self.n_out = torch.empty((1,), dtype=torch.int32, device=dev)
        if mode == "peer":
            import torch.distributed._symmetric_memory as symm

            if self.world > native.MAX_Y_DST:
                raise ValueError(f"peer mode stores to at most {native.MAX_Y_DST} ranks")
            self.Y = symm.empty((T_max, self.N), dtype=dtype, device=dev)
            self.handle = symm.rendezvous(self.Y, group=self._group_name())
            self.dst = peer_destinations(self.Y.data_ptr(), list(self.handle.buffer_ptrs), self.rank)
        else:
            self.Y_shard = torch.empty((T_max, n), dtype=dtype, device=dev)

    def _group_name(self):
        g = self.group if self.group is not None else dist.group.WORLD
        return g.group_name

    def forward(self, X: torch.Tensor, threshold: float) -> torch.Tensor:
        """Y [T, N] (the full output, identical on every rank).  In peer mode the
        result is a view of the layer's symmetric output buffer: the next
        forward overwrites it (clone it to keep it)."""
        T = X.shape[0]
        if T > self.T_max:
            raise ValueError(f"T={T} > T_max={self.T_max}")
        if self.mode == "peer":
            self.handle.barrier(channel=0)  # no rank still reads the previous Y
            native.int8_linear_forward_sharded(X, self.CB, self.SCB, self.bias, threshold, self.dst, self.N, self.lo,
                                               idx=self.idx, n_out=self.n_out, workspace=self.ws, path=self.path)
            self.handle.barrier(channel=0)  # every rank's block has landed everywhere
            return self.Y[:T]
        Ys = self.Y_shard[:T]
        native.int8_linear_forward(X, self.CB, self.SCB, self.bias, threshold, Y=Ys, idx=self.idx,
                                   n_out=self.n_out, workspace=self.ws, path=self.path)
        return gather_columns(Ys, self.group)

    def check_status(self) -> tuple[int, int]:
        return native.int8_check_status(self.ws)
