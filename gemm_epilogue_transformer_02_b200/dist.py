"""Multi-GPU plumbing of the hot path (one process per GPU, torch.distributed).

The block is row-independent: RMSNorm, SwiGLU and the cross-entropy are per
token, so N GPUs run N independent batches (data parallel, weak scaling) with
no collective on the forward data path.  Collectives:

* measurement: a barrier around the timed region and the max over ranks of
  the device time;
* the data-parallel backward (``block_backward_dp``): the weight gradients
  dW2, dW1 and dgamma are sums over tokens, so each is summed over ranks by
  an all-reduce (NCCL over NVLink on GPUs); dW2's all-reduce is issued as
  soon as its GEMM is queued, so it can run while the rest of the backward
  computes;
* the data-parallel cross-entropy (``lmhead_ce_dp``): the global mean needs
  one all-reduce of 8 bytes, a rank's (sum of losses, token count); the
  backward then weighs every token by 1 / global count and sums dW over
  ranks (dH stays with the rank that owns the tokens).

The compute steps go through `ops` (the binding module, or any object with
the same functions), so the orchestration itself holds no arithmetic: every
number is formed by the library's kernels, and the collectives only add.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env():
    """(world_size, rank, local_rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: int = 300):
    """Initialise the process group when launched with more than one rank."""
    ws, rank, local = env()
    if ws > 1 and not dist.is_initialized():
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return ws, rank, local


def rank_seed(base: int, rank: int) -> int:
    """Seed of a rank's own batch (each rank draws different tokens)."""
    return base + 1000 * rank


def barrier():
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(value: float, device=None) -> float:
    """The largest of every rank's value (device time of the timed region)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(work_per_rank_per_step: float, steps: int, max_seconds: float, world: int) -> float:
    """Whole-job throughput: the work of all ranks divided by the slowest rank's time."""
    return world * work_per_rank_per_step * steps / max_seconds


def shutdown():
    if dist.is_available() and dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()


def _active():
    # a one-rank group still runs its collectives (an identity), so that the
    # same calls are exercised on a single GPU
    return dist.is_available() and dist.is_initialized()


def allreduce_sum_async(t, group=None):
    """Starts an in-place sum over ranks of `t`; returns a handle (None without a process group)."""
    if not _active():
        return None
    return dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group, async_op=True)


def wait_all(handles):
    for h in handles:
        if h is not None:
            h.wait()


def allreduce_sum_(tensors, group=None):
    """In-place sum over ranks of every tensor (issued together, then waited)."""
    wait_all([allreduce_sum_async(t, group) for t in tensors])
    return tensors


def block_backward_dp(ops, dOut, x, W1, W2, gamma, fwd, group=None):
    """Backward of the fused block on this rank's tokens, with the weight
    gradients summed over ranks.  dx, dres (= dh) stay per rank.  Returns the
    same dict as ``ops.block_backward``."""
    d_hg, dW2, pdr = ops.gemm_rowscale_bwd(dOut, fwd["hg"], W2, fwd["r"])
    h_w2 = allreduce_sum_async(dW2, group)  # overlaps the rest of the backward
    dh, dgamma = ops.rms_reduce_bwd(pdr, fwd["r"], d_hg, fwd["h"], gamma)
    dx, dW1 = ops.gemm_res_partialrms_bwd(dh, x, W1)
    wait_all([h_w2, allreduce_sum_async(dW1, group), allreduce_sum_async(dgamma, group)])
    return {"dW2": dW2, "dgamma": dgamma, "dh": dh, "dres": dh, "dx": dx, "dW1": dW1, "d_hg": d_hg, "pdr": pdr}


def lmhead_ce_dp(ops, H, W, labels, group=None):
    """Fused LM-head cross-entropy on this rank's tokens with the mean over
    every rank's tokens.  Returns (loss [M], lse [M], global mean [1],
    d_loss [M] = 1 / global token count, the weights of the backward)."""
    loss, lse, _ = ops.lmhead_ce(H, W, labels)
    stats = ops.loss_stats(loss)
    allreduce_sum_([stats], group)
    mean, d_loss = ops.ce_global_finish(stats, H.shape[0])
    return loss, lse, mean, d_loss


def lmhead_ce_bwd_dp(ops, H, W, labels, lse, d_loss, group=None):
    """Backward of the global mean loss: dH for this rank's tokens, dW summed over ranks."""
    dH, dW = ops.lmhead_ce_bwd(H, W, labels, lse, d_loss=d_loss)
    allreduce_sum_([dW], group)
    return dH, dW
