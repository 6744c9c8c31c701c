"""Token-sharded (data-parallel) training step of the TwELL gated FFN.

The FFN acts on every token row independently, so a batch splits by rows: each
rank runs the forward and the backward of its own token shard against the full,
replicated weights, and the only exchange of the step is the sum over ranks of
the weight gradients (dW_g, dW_u, dW_d and db_g; 3 * 4 * d_model * d_ff + 4 * d_ff
bytes). Y and dX stay on the rank that owns the rows. The pages describe a
single-GPU kernel and say nothing on multi-GPU execution; this is the plainest
data-parallel reading of the training step they describe ("Sakana AI и NVIDIA
представили TwELL — формат и CUDA-ядра ...", paragraph 2: training runs on the
hybrid format).

The sum runs as one NCCL all-reduce per gradient tensor over torch.distributed,
issued asynchronously in the order the kernels finish them (the weight
gradients all come out of the last kernel of twell_ffn_bwd), so the exchange
overlaps whatever the caller enqueues next on its compute stream (the backward
of the layer below, in a model); `step(..., wait=False)` returns the handles.
No TMA multicast and no library kernel ever reads a peer's memory here: the
exchange is NCCL's, on this rank's own buffers.

The local compute is the CUDA library (twell_ffn_fwd + twell_ffn_bwd). The
class accepts another local step only so that the sharding and reduction logic
can be exercised on CPU process groups in tests.
"""

from __future__ import annotations

from typing import Callable, Optional

import torch


def shard_bounds(M: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [lo, hi) of a batch of M token rows owned by `rank` of `world`:
    contiguous shards whose sizes differ by at most one row."""
    if world < 1 or not (0 <= rank < world) or M < 0:
        raise ValueError("need world >= 1, 0 <= rank < world and M >= 0")
    base, extra = divmod(M, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


GRAD_KEYS = ("dW_d", "dW_u", "dW_g", "db_g")


def allreduce_grads(grads: dict, group=None, wait: bool = True) -> list:
    """Sums the weight gradients of `grads` over the process group in place, one
    asynchronous all-reduce per tensor in GRAD_KEYS order; returns the pending
    handles (none when wait=True or when the group has one rank). With NCCL a
    handle's wait() makes the current stream wait for the collective."""
    import torch.distributed as dist

    handles = []
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        for k in GRAD_KEYS:
            handles.append(dist.all_reduce(grads[k], op=dist.ReduceOp.SUM, group=group, async_op=True))
    if wait:
        for h in handles:
            h.wait()
        return []
    return handles


class ShardedTwellFFN:
    """One data-parallel training step per call: local TwELL forward and backward
    on this rank's rows, then the weight gradients summed over the process group.

    Buffers (state, workspaces, outputs) are allocated on first use for a given
    shape and reused, so repeated steps allocate nothing.
    """

    def __init__(self, group=None, T_n: int = 128, K: int = 8, ovf_cap: Optional[int] = None,
                 dense_min: int = 0, local_step: Optional[Callable] = None):
        self.group = group
        self.T_n, self.K, self.ovf_cap, self.dense_min = T_n, K, ovf_cap, dense_min
        self._local = local_step
        self._bufs = None
        self._key = None

    def _cuda_step(self, X, W_g, b_g, W_u, W_d, dY, lam):
        from . import HybridState, OP_BWD, OP_FWD, ffn_bwd, ffn_fwd, transpose_wd, workspace

        M, d = X.shape
        f = W_g.shape[0]
        key = (M, d, f, X.device)
        if self._key != key:
            cap = M if self.ovf_cap is None else min(int(self.ovf_cap), M)
            dev = X.device
            self._bufs = dict(
                st=HybridState(M, f, self.T_n, self.K, cap, dev, with_u=True, dense_min=self.dense_min),
                wsf=workspace(OP_FWD, M, d, f, self.T_n, self.K, cap, dev),
                wsb=workspace(OP_BWD, M, d, f, self.T_n, self.K, cap, dev),
                Wdt=torch.empty((f, d), dtype=torch.bfloat16, device=dev),
                Y=torch.empty((M, d), dtype=torch.bfloat16, device=dev),
                out=dict(dX=torch.empty((M, d), device=dev), dW_g=torch.empty((f, d), device=dev),
                         dW_u=torch.empty((f, d), device=dev), dW_d=torch.empty((d, f), device=dev),
                         db_g=torch.empty(f, device=dev)))
            self._key = key
        b = self._bufs
        transpose_wd(W_d, out=b["Wdt"])
        ffn_fwd(X, W_g, b_g, W_u, W_d, T_n=self.T_n, K=self.K, W_dt=b["Wdt"], state=b["st"], ws=b["wsf"], Y=b["Y"])
        g = ffn_bwd(X, W_g, W_u, W_d, b["st"], dY, lam=lam, W_dt=b["Wdt"], ws=b["wsb"], out=b["out"])
        return dict(Y=b["Y"], **g)

    @property
    def state(self):
        """The hybrid state of the last local forward (CUDA path only)."""
        return None if self._bufs is None else self._bufs["st"]

    def step(self, X, W_g, b_g, W_u, W_d, dY, lam: float = 0.0, wait: bool = True):
        """Forward + backward of this rank's rows X [M_local, d_model] with the
        replicated weights, loss sum(Y * dY) + lam * sum(ReLU(z)) over the whole
        batch. Returns (out, handles): out holds this rank's Y and dX and the
        weight gradients summed over the group (valid once the handles have
        completed; wait=True waits for them)."""
        out = (self._local or self._cuda_step)(X, W_g, b_g, W_u, W_d, dY, lam)
        return out, allreduce_grads(out, self.group, wait)
