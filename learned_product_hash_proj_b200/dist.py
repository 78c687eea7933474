"""One process per GPU: rank discovery, the host-side aggregation of a
multi-GPU measurement, and the head-sharded mixer.

The mixer's work shards with no exchange: every (batch, head) routes and
attends on its own, so N GPUs run N independent replicas of a workload (each
rank its own sequences) and the only collective is the reduction of the
timings (the maximum over ranks) and of the token counts (the sum).

Head sharding splits one workload instead: rank r of N runs the heads
[r H/N, (r+1) H/N) -- their rows of Wq, Wk, Wv, their columns of Wo and their
codebooks -- through the whole mixer.  Projection, routing (codebooks, posting
lists and probes are per head) and attention of a head need nothing from the
other heads; the output projection delta = sum_h O_h Wo_h^T leaves each rank a
partial sum over its heads, and one all-reduce (sum) gives every rank delta.
head_sharded_forward_fused replaces that all-reduce by the output projection
fused with a reduce-scatter over peer memory (fp32 partials, one rounding).
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env_rank() -> tuple[int, int, int]:
    """(rank, local_rank, world_size) from the torchrun environment (defaults 0, 0, 1)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def init(backend: str = "nccl", timeout_s: float = 120.0) -> tuple[int, int, int]:
    """Join the process group when WORLD_SIZE > 1 (MASTER_ADDR/PORT from the env)."""
    rank, local, world = env_rank()
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=timeout_s))
    return rank, local, world


def barrier():
    if dist.is_initialized():
        dist.barrier()


def reduce_max(values, device="cpu") -> list[float]:
    """Elementwise maximum over ranks of a list of floats."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_initialized():
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def reduce_sum(values, device="cpu") -> list[float]:
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_initialized():
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return t.tolist()


def replica_seed(seed: int, rank: int) -> int:
    """Each rank's replica draws its own sequences."""
    return int(seed) * 1009 + int(rank)


def throughput(tokens_per_rank: list[float], seconds_per_rank: list[float], device="cpu") -> float:
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's time."""
    tot = reduce_sum([sum(tokens_per_rank)], device)[0]
    t = reduce_max([max(seconds_per_rank)], device)[0]
    return tot / t


# --- head-sharded mixer ----------------------------------------------------


def head_range(H: int, rank: int, world: int) -> tuple[int, int]:
    """The heads [h0, h1) of `rank` when H heads are split evenly over `world` ranks."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if H % world:
        raise ValueError(f"{H} heads do not split evenly over {world} ranks")
    per = H // world
    return rank * per, (rank + 1) * per


def shard_config(cfg, rank: int, world: int):
    """The configuration one rank runs: the same workload with its H / world heads."""
    h0, h1 = head_range(cfg.H, rank, world)
    return cfg.with_(H=h1 - h0)


def _contig(a):
    return a.contiguous() if isinstance(a, torch.Tensor) else a.copy()


def shard_weights(params: dict, cfg, rank: int, world: int) -> dict:
    """Rank's slice of the mixer's parameters (numpy arrays or torch tensors, copied contiguous):
    rows [h0 d, h1 d) of Wq, Wk, Wv ([H d, W]), the same columns of Wo ([W, H d]) and heads
    [h0, h1) of the codebooks ([H, M, C, d/M]).  Other entries (x) are passed through."""
    h0, h1 = head_range(cfg.H, rank, world)
    r0, r1 = h0 * cfg.d, h1 * cfg.d
    out = dict(params)
    for k in ("Wq", "Wk", "Wv"):
        out[k] = _contig(params[k][r0:r1])
    out["Wo"] = _contig(params["Wo"][:, r0:r1])
    out["codebooks"] = _contig(params["codebooks"][h0:h1])
    return out


def reduce_partial_delta(delta, group=None, stream=None):
    """Sum the ranks' partial deltas in place: every rank ends with the whole delta.  The sum is
    taken in delta's dtype (for bf16 storage each reduction step rounds to bf16).  With a CUDA
    stream, the all-reduce is ordered after the work already queued on it."""
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return delta
    if stream is not None:
        with torch.cuda.stream(stream):
            dist.all_reduce(delta, op=dist.ReduceOp.SUM, group=group)
    else:
        dist.all_reduce(delta, op=dist.ReduceOp.SUM, group=group)
    return delta


def head_sharded_forward(plan, x, shard: dict, delta, ws, group=None, forced=None, stream=None):
    """The mixer on this rank's heads (plan built from shard_config, shard from shard_weights, on
    this rank's GPU), then the all-reduce of the partial delta: delta [B, S, W] is the whole
    mixer's output on every rank.  forced, if given, holds this rank's heads."""
    from . import mono
    mono.forward(plan, x, shard["Wq"], shard["Wk"], shard["Wv"], shard["Wo"], shard["codebooks"], delta, ws,
                 forced=forced, stream=stream)
    return reduce_partial_delta(delta, group, stream)


# --- head-sharded mixer, output projection fused with the reduce-scatter ----


def stage_rows(cfg, world: int) -> int:
    """Token rows per rank in the reduce-scatter of the head-sharded delta: B*S split into `world` chunks."""
    rows = cfg.B * cfg.S
    if world < 1 or rows % world:
        raise ValueError(f"{rows} token rows do not split evenly over {world} ranks")
    return rows // world


def chunk_of(cfg, world: int, rank: int) -> slice:
    """The rows [rank * rows, (rank + 1) * rows) of the flattened [B*S, W] delta that `rank` reduces."""
    rows = stage_rows(cfg, world)
    return slice(rank * rows, (rank + 1) * rows)


def alloc_stage(cfg, world: int, device, symmetric: bool = False, group=None):
    """This rank's staging buffer [world, rows, W] fp32 for the partials the ranks send it.  With
    `symmetric`, the buffer comes from torch's symmetric memory and the return value also lists every rank's
    buffer as a device address this GPU can store to (NVLink peer access); else only the local buffer."""
    shape = (world, stage_rows(cfg, world), cfg.W)
    if not symmetric:
        return torch.empty(shape, dtype=torch.float32, device=device), None
    import torch.distributed._symmetric_memory as symm_mem
    buf = symm_mem.empty(shape, dtype=torch.float32, device=device)
    hdl = symm_mem.rendezvous(buf, group if group is not None else dist.group.WORLD)
    return buf, [int(p) for p in hdl.buffer_ptrs]


def head_sharded_forward_fused(plan, x, shard: dict, delta, ws, stage, stage_ptrs, rank: int, world: int,
                               group=None, forced=None, stream=None):
    """The mixer on this rank's heads with the output projection fused into the reduce-scatter: the GEMM
    epilogue stores each fp32 row of the partial delta into the staging buffer of the rank that owns the row
    (stage_ptrs, every rank's buffer from alloc_stage(symmetric=True)); a collective on the stream then orders
    every rank's stores before this rank sums the `world` partials of its rows in fp32, in rank order, and
    rounds once; an all-gather gives every rank the whole delta [B, S, W]."""
    from . import mono
    cfg = plan.cfg
    Q, K, V, sel, O = (plan.region(ws, k) for k in ("Q", "K", "V", "sel", "O"))
    mono.project(plan, x, shard["Wq"], shard["Wk"], shard["Wv"], Q, K, V, ws, stream)
    mono.route(plan, Q, K, shard["codebooks"], sel, ws, forced=forced, stream=stream)
    mono.attend(plan, Q, K, V, sel, O, ws, stream)
    mono.out_project_scatter(plan, O, shard["Wo"], stage_ptrs, rank, ws, stream)
    flat = delta.view(-1, cfg.W)
    chunk = torch.empty_like(flat[chunk_of(cfg, world, rank)])
    ctx = torch.cuda.stream(stream) if stream is not None else _null()
    with ctx:
        if dist.is_initialized() and world > 1:
            dist.all_reduce(torch.zeros(1, device=delta.device), group=group)   # every rank's stores are done
        mono.stage_reduce(plan, stage, world, chunk, stream)
        if dist.is_initialized() and world > 1:
            dist.all_gather_into_tensor(flat, chunk, group=group)
        else:
            flat.copy_(chunk)
    return delta


class _null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def finalize():
    if dist.is_initialized():
        dist.destroy_process_group()
