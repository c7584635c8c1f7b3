"""One GPTQ layer spread over the ranks of a process group.

"GPTQ / AWQ / SqueezeLLM" sec. 一 builds H from the calibration inputs, a sum
over tokens; the loop of "INT4/INT8 量化推理" sec. 三 treats every output row
on its own once the factor of H^-1 is fixed.  So a layer splits as:

  rank r   S_r = X_r^T X_r over its share of the tokens    gptq_hessian_accumulate
  all      S = sum_r S_r                                    one all-reduce (the only exchange)
  all      perm, U from S, the same on every rank           gptq_prepare_hinv
  rank r   its share of W's rows quantized and packed       gptq_quantize_layer, gptq_pack_int4

The all-reduce goes through torch.distributed (NCCL between GPUs) on the
current stream, and every rank makes the same calls in the same order.  The
preparation is repeated on every rank rather than broadcast: it needs only S,
and a broadcast of U would be a second exchange of the same size as S.
"""
from __future__ import annotations

import torch

from . import gptq as G


def share(total: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous [lo, hi) of `total` items for `rank`: equal parts, the first
    total % world ranks one item more."""
    if world < 1 or not 0 <= rank < world or total < 0:
        raise ValueError("bad share arguments")
    q, r = divmod(total, world)
    lo = rank * q + min(rank, r)
    return lo, lo + q + (1 if rank < r else 0)


def _world(group):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(group), dist.get_rank(group)
    return 1, 0


class ShardedLayer:
    """Buffers and one pass of a d_out x d_in layer over the group's ranks.

    n_local: this rank's calibration tokens (the ranks' counts may differ).
    The rank's rows are rows[0]:rows[1] of W; step() takes exactly those rows
    and this rank's tokens and leaves the rank's codes, scales, zeros,
    row_loss, qweight and qzeros in the attributes of the same names.
    """

    def __init__(self, d_out: int, d_in: int, n_local: int, device, group=None, bits: int = 4,
                 group_size: int = 128, act_order: bool = False, damp_rel: float = 0.01):
        self.group = group
        self.world, self.rank = _world(group)
        self.m, self.d = int(d_out), int(d_in)
        self.rows = share(self.m, self.world, self.rank)
        self.bits, self.group_size = int(bits), int(group_size)
        self.act_order, self.damp_rel = bool(act_order), float(damp_rel)
        dev = torch.device(device)
        d, mr = self.d, self.rows[1] - self.rows[0]
        self.n_local = int(n_local)
        self.n_total = self._sum_over_ranks(self.n_local, dev)
        if self.n_total <= 0:
            raise ValueError("no calibration tokens on any rank")
        self.S = torch.zeros(d, d, dtype=torch.float32, device=dev)
        self.perm = torch.empty(d, dtype=torch.int32, device=dev)
        self.U = torch.empty(d, d, dtype=torch.float32, device=dev)
        self.info = torch.zeros(1, dtype=torch.int32, device=dev)
        self.ws_p = torch.empty(G.gptq_prepare_workspace_bytes(d), dtype=torch.uint8, device=dev)
        ng = d // self.group_size
        self.codes = torch.empty(mr, d, dtype=torch.uint8, device=dev)
        self.scales = torch.empty(mr, ng, dtype=torch.float16, device=dev)
        self.zeros = torch.empty(mr, ng, dtype=torch.uint8, device=dev)
        self.row_loss = torch.empty(mr, dtype=torch.float32, device=dev)
        self.ws_q = torch.empty(G.gptq_quantize_workspace_bytes(max(mr, 1), d, 128),
                                dtype=torch.uint8, device=dev)
        self.qweight = torch.empty(mr, d // 8, dtype=torch.int32, device=dev)
        self.qzeros = torch.empty(mr, (ng + 1) // 2, dtype=torch.uint8, device=dev)

    def _sum_over_ranks(self, v: int, dev) -> int:
        if self.world == 1:
            return int(v)
        import torch.distributed as dist
        t = torch.tensor([v], dtype=torch.int64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=self.group)
        return int(t.item())

    def hessian(self, X_local: torch.Tensor):
        """S = sum over all ranks' tokens of X^T X (upper triangle)."""
        if X_local.shape != (self.n_local, self.d):
            raise ValueError("X_local must be n_local x d_in")
        self.S.zero_()
        if self.n_local:
            G.gptq_hessian_accumulate(self.S, X_local)
        if self.world > 1:
            import torch.distributed as dist
            dist.all_reduce(self.S, op=dist.ReduceOp.SUM, group=self.group)

    def hessian_from_host(self, streamer, X_host: torch.Tensor):
        """hessian() for this rank's tokens held in host memory, streamed
        through a gptq.HostHessian (its PCIe copies overlap the accumulation)."""
        if X_host.shape != (self.n_local, self.d):
            raise ValueError("X_host must be n_local x d_in")
        self.S.zero_()
        if self.n_local:
            streamer.accumulate(self.S, X_host)
        if self.world > 1:
            import torch.distributed as dist
            dist.all_reduce(self.S, op=dist.ReduceOp.SUM, group=self.group)

    def quantize(self, W_rows: torch.Tensor):
        """perm and U from the summed S, then this rank's rows."""
        lo, hi = self.rows
        if W_rows.shape != (hi - lo, self.d):
            raise ValueError("W_rows must be this rank's rows of W")
        G.gptq_prepare_hinv(self.S, self.n_total, self.damp_rel, self.act_order, self.perm,
                            self.U, self.info, self.ws_p)
        if hi == lo:
            return
        G.gptq_quantize_layer(W_rows, self.U, self.perm if self.act_order else None, self.bits,
                              self.group_size, 128, self.codes, self.scales, self.zeros,
                              self.row_loss, self.ws_q)
        if self.bits == 4:
            G.gptq_pack_int4(self.codes, self.zeros, self.qweight, self.qzeros)

    def step(self, W_rows: torch.Tensor, X_local: torch.Tensor):
        self.hessian(X_local)
        self.quantize(W_rows)
