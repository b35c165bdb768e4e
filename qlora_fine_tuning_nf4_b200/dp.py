"""Data-parallel plumbing for the gated-MLP step: token sharding and the one
exchange the path has, the sum of the LoRA gradients across ranks.

Tokens are independent for Y, dX and the activations, so each rank runs its own
batch; only dA and dB are sums over tokens, so data-parallel training all-reduces
them (the pages' DDP runs do the same gradient sync).  The six adapter
gradients live as views of one flat buffer so one collective moves them all.
"""

import torch
import torch.distributed as dist

GRAD_ORDER = ("dA_g", "dB_g", "dA_u", "dB_u", "dA_d", "dB_d")


def grad_shapes(d, h, r):
    return {"dA_g": (d, r), "dB_g": (r, h), "dA_u": (d, r), "dB_u": (r, h), "dA_d": (h, r), "dB_d": (r, d)}


def flat_lora_grads(d, h, r, device, dtype=torch.bfloat16):
    """One flat buffer and its six contiguous, 16-byte aligned views."""
    shapes = grad_shapes(d, h, r)
    total = sum(a * b for a, b in shapes.values())
    flat = torch.empty(total, dtype=dtype, device=device)
    views, off = {}, 0
    for name in GRAD_ORDER:
        a, b = shapes[name]
        views[name] = flat[off:off + a * b].view(a, b)
        off += a * b
    return flat, views


def shard_rows(M_total, rank, world):
    """Contiguous token range [lo, hi) of this rank."""
    per = (M_total + world - 1) // world
    lo = min(M_total, rank * per)
    return lo, min(M_total, lo + per)


def allreduce_lora_grads(flat, group=None):
    """Sum the flat gradient buffer over all ranks (in place)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    return flat
