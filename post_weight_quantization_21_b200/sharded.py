"""One layer solved across the ranks of a process group (one process per GPU).

The layer's work splits the way the method allows (FDE Interviews breakdown of GPTQ, section 01: the
objective's curvature H = 2 X X^T is a sum over calibration tokens, and a fixed column order lets
every row share one inverse-Hessian computation):

* Hessian: tokens are sharded.  Rank r accumulates H_r = 2 X_r^T X_r over its token range, then one
  all-reduce (sum) over the process group gives every rank the full H.  Only the upper triangle is
  meaningful; the all-reduce moves the whole d x d buffer in row panels (the strict lower part is
  summed along and never read).
* Prepare: U = chol((H + lambda I)^-1) is the same on every rank.  Either every rank computes it from
  its identical copy of H ("replicated": the all-reduce leaves bit-identical H everywhere and the
  kernels are deterministic), or rank 0 computes it and broadcasts it ("broadcast").
* Solve: rows are sharded.  Rows are independent given U, so rank r quantizes and packs its own rows
  with no exchange.  The results stay sharded (each rank owns its rows' packed codes and grids);
  ``gather_results`` collects them on every rank when asked.

The compute steps are injected (``ops``): the product uses the CUDA library through the binding on
each rank's GPU (``cuda_ops``); tests run the same partitioning with gloo on CPU with other compute
functions.  Nothing here computes any part of the method itself: it only splits, moves and joins
buffers.
"""
from __future__ import annotations

import dataclasses
from typing import Callable

import torch
import torch.distributed as dist


def shard_range(n: int, world: int, rank: int, align: int = 1) -> tuple[int, int]:
    """[lo, hi) of rank's share of n items: contiguous, in rank order, each boundary a multiple of
    ``align`` (the last rank takes the remainder)."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad rank / world")
    units = (n + align - 1) // align
    per, extra = divmod(units, world)
    lo_u = rank * per + min(rank, extra)
    hi_u = lo_u + per + (1 if rank < extra else 0)
    return min(lo_u * align, n), min(hi_u * align, n)


@dataclasses.dataclass
class ShardOps:
    """The four compute steps, each on this rank's tensors (in place into the given outputs)."""
    hessian: Callable        # (X_local, H) -> None            H = 2 X_local^T X_local (upper valid)
    prepare: Callable        # (H, U) -> None                  U = chol((H + damp mean(diag H) I)^-1)
    quantize: Callable       # (W_local, U, codes, scales, zeros) -> None
    pack: Callable           # (codes, packed) -> None


def cuda_ops(solver_cfg: dict, device) -> ShardOps:
    """ShardOps over the CUDA library (the binding's calls on this rank's GPU)."""
    import post_weight_quantization_21_b200 as g
    bits, gs, B, damp = solver_cfg["bits"], solver_cfg["group_size"], solver_cfg["block_size"], solver_cfg["damp"]
    m_local, d, n_local = solver_cfg["m_local"], solver_cfg["d"], solver_cfg["n_local"]
    x_dtype, flags = solver_cfg["x_dtype"], solver_cfg.get("flags", 0)
    ws_bytes = max(g.gptq_hessian_workspace_size(max(n_local, 1), d, x_dtype), g.gptq_prepare_workspace_size(d),
                   g.gptq_quantize_workspace_size(max(m_local, 1), d, bits, gs, B), 256)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device)
    status = torch.zeros(3, 2, dtype=torch.int32, device=device)

    def hessian(X, H):
        g.gptq_hessian_accumulate(X, H, status[0], ws, 2.0, False)

    def prepare(H, U):
        g.gptq_prepare_uinv(H, U, status[1], ws, damp)

    def quantize(W, U, codes, scales, zeros):
        if W.shape[0]:
            g.gptq_quantize_layer(W, U, codes, scales, zeros, status[2], ws, bits, gs, B, flags)

    def pack(codes, packed):
        if codes.shape[0]:
            g.gptq_pack(codes, bits, packed)

    ops = ShardOps(hessian, prepare, quantize, pack)
    ops.status = status
    return ops


class ShardedLayerSolver:
    """Buffers of this rank's share of one layer and the partitioned solve (see the module notes).

    X_local: this rank's tokens [n_local, d]; W_local: this rank's rows [m_local, d].  H and U are
    full d x d on every rank.  ``run()`` leaves this rank's codes / scales / zeros / packed filled.
    """

    PANEL_ROWS = 4096  # rows of H per all-reduce call (bounds the size of one collective)

    def __init__(self, m: int, d: int, n_tokens: int, bits: int, group_size: int, block_size: int, damp: float,
                 x_dtype, w_dtype, device, ops: ShardOps | None = None, group=None, u_source: str = "replicated",
                 token_align: int = 64, h_dtype=torch.float32):
        if u_source not in ("replicated", "broadcast"):
            raise ValueError(u_source)
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.m, self.d, self.n_tokens = m, d, n_tokens
        self.bits, self.group_size, self.block_size, self.damp = bits, group_size, block_size, damp
        self.u_source = u_source
        self.tokens = shard_range(n_tokens, self.world, self.rank, token_align)
        self.rows = shard_range(m, self.world, self.rank)
        n_local = self.tokens[1] - self.tokens[0]
        m_local = self.rows[1] - self.rows[0]
        n_groups = 1 if group_size == 0 else d // group_size
        dev = torch.device(device)
        self.X_local = torch.empty(n_local, d, dtype=x_dtype, device=dev)
        self.W_local = torch.empty(m_local, d, dtype=w_dtype, device=dev)
        self.H = torch.empty(d, d, dtype=h_dtype, device=dev)
        self.U = torch.empty_like(self.H)
        self.codes = torch.empty(m_local, d, dtype=torch.uint8, device=dev)
        self.scales = torch.empty(m_local, n_groups, dtype=torch.float32, device=dev)
        self.zeros = torch.empty(m_local, n_groups, dtype=torch.int32, device=dev)
        self.packed = torch.empty(m_local, d * bits // 32, dtype=torch.int32, device=dev)
        if ops is None:
            ops = cuda_ops({"bits": bits, "group_size": group_size, "block_size": block_size, "damp": damp,
                            "m_local": m_local, "d": d, "n_local": n_local, "x_dtype": x_dtype}, dev)
        self.ops = ops

    # ------------------------------------------------------------------------------ steps
    def hessian(self):
        """Local H over this rank's tokens, then the sum over ranks (every rank ends with the full H)."""
        self.ops.hessian(self.X_local, self.H)
        if self.world > 1:
            for r0 in range(0, self.d, self.PANEL_ROWS):
                dist.all_reduce(self.H[r0:r0 + self.PANEL_ROWS], op=dist.ReduceOp.SUM, group=self.group)

    def prepare(self):
        if self.world == 1 or self.u_source == "replicated":
            self.ops.prepare(self.H, self.U)
            return
        if self.rank == 0:
            self.ops.prepare(self.H, self.U)
        for r0 in range(0, self.d, self.PANEL_ROWS):
            dist.broadcast(self.U[r0:r0 + self.PANEL_ROWS], src=self._global_rank(0), group=self.group)

    def quantize(self):
        self.ops.quantize(self.W_local, self.U, self.codes, self.scales, self.zeros)

    def pack(self):
        self.ops.pack(self.codes, self.packed)

    def run(self):
        self.hessian()
        self.prepare()
        self.quantize()
        self.pack()

    def check_status(self):
        """Raises GPTQError with the first failure this rank's calls recorded on the device."""
        status = getattr(self.ops, "status", None)
        if status is None:
            return
        import post_weight_quantization_21_b200 as g
        for word in status:
            code, detail = g.gptq_read_status(word)
            if code != g.GPTQ_OK:
                raise g.GPTQError(code, "device status", detail)

    def run_host(self, W_host, X_host, out_packed, out_scales, out_zeros):
        """This rank's shares through host memory: its rows of W and its tokens of X copied in (pinned
        host tensors for asynchronous copies), the partitioned solve, its rows' results copied out."""
        self.W_local.copy_(W_host, non_blocking=True)
        self.X_local.copy_(X_host, non_blocking=True)
        self.run()
        out_packed.copy_(self.packed, non_blocking=True)
        out_scales.copy_(self.scales, non_blocking=True)
        out_zeros.copy_(self.zeros, non_blocking=True)

    # ------------------------------------------------------------------------------ results
    def gather_results(self):
        """(codes, scales, zeros, packed) of all m rows on every rank, in row order."""
        out = []
        for t in (self.codes, self.scales, self.zeros, self.packed):
            if self.world == 1:
                out.append(t)
                continue
            counts = [shard_range(self.m, self.world, r)[1] - shard_range(self.m, self.world, r)[0]
                      for r in range(self.world)]
            width = t.shape[1]
            pad = max(counts)
            buf = torch.zeros(pad, width, dtype=t.dtype, device=t.device)
            buf[:t.shape[0]] = t
            parts = [torch.empty_like(buf) for _ in range(self.world)]
            dist.all_gather(parts, buf, group=self.group)
            out.append(torch.cat([p[:c] for p, c in zip(parts, counts)]))
        return tuple(out)

    def _global_rank(self, group_rank: int) -> int:
        if self.group is None:
            return group_rank
        return dist.get_global_rank(self.group, group_rank)
