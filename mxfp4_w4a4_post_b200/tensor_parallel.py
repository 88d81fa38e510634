"""Tensor-parallel MACaQ W4A4 linear layers over torch.distributed (NCCL between B200s).

Two shardings of y = x W^T, W [N, K]:

* column-parallel: rank r holds rows n0 .. n1 - 1 of W (so of W' = W diag(s) Hb, whose
  quantisation is row by row); it computes y[:, n0:n1] with the unchanged layer and one
  all-gather joins the columns (or the caller keeps the shard).
* row-parallel: rank r holds the K range k0 .. k1 - 1, cut on 32-element boundaries.
  The rotation Hb is block-diagonal with 32 x 32 blocks aligned with the MX blocks and
  diag(s) is per channel, so a shard's transform, E8M0 scales and E2M1 codes are exactly
  the corresponding columns of the unsharded ones (MACaQ articles: the transform section
  and the MX format section, 32-element blocks sharing one E8M0 scale). Each rank
  computes an fp32 partial product over its K range and one all-reduce (sum) gives y.

All arithmetic runs in the library's kernels through the package's binding; this module
cuts the weight, picks each rank's slice of x and issues the one collective. The
per-rank operations are an object with `prepare(W, s)`, `linear(x, w, out_dtype)` and
`linear_gather(x, w, dests)`; the default is the CUDA binding.

The column cut can also skip the collective: `ColumnParallelW4A4.forward_into` hands
the GEMM every rank's full-width y (as this process sees it: its own buffer and the
other GPUs' buffers mapped into it), and the GEMM's epilogue writes this rank's columns
into all of them (`macaq_linear_w4a4_gather`). The caller orders the writes with the
readers (for example a barrier on every rank's stream afterwards).
"""
from dataclasses import dataclass

MX_BLOCK = 32


def split_range(n, world, rank, align=1):
    """[lo, hi) of rank `rank` when n items, in units of `align`, are cut into `world`
    contiguous pieces whose sizes differ by at most one unit (the first ranks get the
    larger pieces; the last unit may be partial). Pieces may be empty."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad rank {rank} of {world}")
    if n < 0 or align < 1:
        raise ValueError("bad size")
    units = -(-n // align)
    base, extra = divmod(units, world)
    lo_u = rank * base + min(rank, extra)
    hi_u = lo_u + base + (1 if rank < extra else 0)
    return min(lo_u * align, n), min(hi_u * align, n)


def split_k(K, world, rank):
    """K range of a row-parallel rank: whole 32-element MX blocks."""
    if K % MX_BLOCK:
        raise ValueError(f"K={K} is not a multiple of {MX_BLOCK}")
    return split_range(K, world, rank, MX_BLOCK)


class CudaOps:
    """The library's kernels, through the Python binding."""

    def prepare(self, W, s):
        import mxfp4_w4a4_post_b200 as mq
        return mq.prepare_weight(W, s)

    def linear(self, x, w, out_dtype):
        import mxfp4_w4a4_post_b200 as mq
        return mq.linear(x, w, out_dtype=out_dtype)

    def linear_gather(self, x, w, dests):
        import mxfp4_w4a4_post_b200 as mq
        return mq.linear_gather(x, w, dests)


def _dist():
    import torch.distributed as dist
    return dist


def _in_group():
    dist = _dist()
    return dist.is_available() and dist.is_initialized()


def _world(group):
    if _in_group():
        dist = _dist()
        return dist.get_world_size(group), dist.get_rank(group)
    return 1, 0


@dataclass
class ColumnParallelW4A4:
    """Rank's rows n0 .. n1 - 1 of the prepared weight."""
    N: int
    K: int
    n0: int
    n1: int
    weight: object          # the ops' prepared weight of W[n0:n1], or None for an empty shard
    group: object = None
    ops: object = None

    def __post_init__(self):
        if self.ops is None:
            self.ops = CudaOps()

    @classmethod
    def from_full(cls, W, s, group=None, ops=None):
        """Cut the full bf16 weight W [N, K] (same on every rank) and prepare this rank's rows."""
        ops = ops or CudaOps()
        world, rank = _world(group)
        N, K = W.shape
        n0, n1 = split_range(N, world, rank)
        w = ops.prepare(W[n0:n1], s) if n1 > n0 else None
        return cls(N, K, n0, n1, w, group, ops)

    def forward(self, x, out_dtype=None, gather=True):
        """x [M, K] (replicated). Returns y [M, N] (gather=True) or this rank's y[:, n0:n1]."""
        import torch
        out_dtype = out_dtype or torch.bfloat16
        M = x.shape[0]
        if self.weight is not None:
            y_local = self.ops.linear(x, self.weight, out_dtype)
        else:
            y_local = torch.empty((M, 0), dtype=out_dtype, device=x.device)
        if not gather or not _in_group():
            return y_local
        world, _ = _world(self.group)
        # pieces differ by at most one column: pad to the widest, gather, trim
        widths = [split_range(self.N, world, r) for r in range(world)]
        wmax = max(hi - lo for lo, hi in widths)
        buf = torch.zeros((M, wmax), dtype=out_dtype, device=x.device)
        buf[:, :y_local.shape[1]] = y_local
        parts = [torch.empty_like(buf) for _ in range(world)]
        _dist().all_gather(parts, buf.contiguous(), group=self.group)
        return torch.cat([p[:, :hi - lo] for p, (lo, hi) in zip(parts, widths)], dim=1)

    def forward_into(self, x, ys):
        """x [M, K] (replicated); ys: full-width outputs [M, N] (one dtype, unit column
        stride, one common row stride), typically every rank's y as mapped into this
        process. Writes this rank's columns n0 .. n1 - 1 of y into each of them with one
        layer call and no collective; returns ys."""
        if self.weight is not None:
            self.ops.linear_gather(x, self.weight, [y[:, self.n0:self.n1] for y in ys])
        return ys


@dataclass
class RowParallelW4A4:
    """Rank's K range k0 .. k1 - 1 (whole MX blocks) of the prepared weight."""
    N: int
    K: int
    k0: int
    k1: int
    weight: object          # the ops' prepared weight of W[:, k0:k1] with s[k0:k1], or None
    group: object = None
    ops: object = None

    def __post_init__(self):
        if self.ops is None:
            self.ops = CudaOps()

    @classmethod
    def from_full(cls, W, s, group=None, ops=None):
        """Cut the full bf16 weight W [N, K] and scale s [K] (same on every rank)."""
        ops = ops or CudaOps()
        world, rank = _world(group)
        N, K = W.shape
        k0, k1 = split_k(K, world, rank)
        w = ops.prepare(W[:, k0:k1], s[k0:k1]) if k1 > k0 else None
        return cls(N, K, k0, k1, w, group, ops)

    def forward(self, x, out_dtype=None):
        """x: [M, K] (replicated; this rank reads columns k0 .. k1 - 1) or [M, k1 - k0]
        (already this rank's slice). Returns y [M, N] on every rank: the fp32 partial
        products summed by one all-reduce, then cast to out_dtype."""
        import torch
        out_dtype = out_dtype or torch.bfloat16
        M, kx = x.shape
        if kx == self.K:
            x_local = x[:, self.k0:self.k1]
        elif kx == self.k1 - self.k0:
            x_local = x
        else:
            raise ValueError(f"x has {kx} columns; expected {self.K} or {self.k1 - self.k0}")
        if self.weight is not None:
            y = self.ops.linear(x_local, self.weight, torch.float32)
        else:
            y = torch.zeros((M, self.N), dtype=torch.float32, device=x.device)
        if _in_group():
            _dist().all_reduce(y, op=_dist().ReduceOp.SUM, group=self.group)
        return y if out_dtype == torch.float32 else y.to(out_dtype)
