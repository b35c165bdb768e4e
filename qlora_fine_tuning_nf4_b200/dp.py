"""Data-parallel plumbing for the QLoRA step: token sharding and the one
exchange the path has, the sum of the LoRA gradients across ranks.

Tokens are independent for Y, dX and the activations, so each rank runs its own
batch; only dA and dB are sums over tokens, so data-parallel training all-reduces
them (the pages' DDP runs do the same gradient sync).  The adapter gradients
live as views of one flat buffer so that few collectives move them all.

In the gated MLP's backward, four of the six adapter gradients (dA_d, dB_d,
dB_g, dB_u) are final before the gate/up dX GEMM, the step's second-largest
kernel, starts; the library records an event at that point
(qlora_mlp_bwd_ev).  Their all-reduce then runs on a side stream while that
GEMM computes, and only dA_g, dA_u are summed after the backward.  The flat
buffer puts the early four first so that each part is one contiguous slice.
"""

import torch
import torch.distributed as dist

# MLP adapter gradients in buffer order: the four final before the gate/up dX GEMM first
GRAD_ORDER = ("dA_d", "dB_d", "dB_g", "dB_u", "dA_g", "dA_u")
MLP_EARLY = 4


def grad_shapes(d, h, r):
    return {"dA_g": (d, r), "dB_g": (r, h), "dA_u": (d, r), "dB_u": (r, h), "dA_d": (h, r), "dB_d": (r, d)}


def flat_buffer(named_shapes, device, dtype=torch.bfloat16):
    """One flat buffer holding each (name, shape) in order as a contiguous view;
    every view starts on a 16-byte boundary (sizes padded to 16 bytes).
    Returns (flat, views, offsets) with offsets[name] = first element."""
    per16 = 16 // torch.tensor([], dtype=dtype).element_size()
    offs, off = {}, 0
    for name, shape in named_shapes:
        n = 1
        for s in shape:
            n *= s
        offs[name] = off
        off += -(-n // per16) * per16
    flat = torch.zeros(off, dtype=dtype, device=device)
    views = {}
    for name, shape in named_shapes:
        n = 1
        for s in shape:
            n *= s
        views[name] = flat[offs[name]:offs[name] + n].view(*shape)
    return flat, views, offs


def flat_lora_grads(d, h, r, device, dtype=torch.bfloat16):
    """The six MLP adapter gradients as views of one flat buffer (GRAD_ORDER).
    Returns (flat, views, early) with flat[:early] the four early gradients."""
    shapes = grad_shapes(d, h, r)
    flat, views, offs = flat_buffer([(k, shapes[k]) for k in GRAD_ORDER], device, dtype)
    return flat, views, offs[GRAD_ORDER[MLP_EARLY]]


def shard_rows(M_total, rank, world):
    """Contiguous token range [lo, hi) of this rank."""
    per = (M_total + world - 1) // world
    lo = min(M_total, rank * per)
    return lo, min(M_total, lo + per)


def allreduce_lora_grads(flat, group=None):
    """Sum the flat gradient buffer over all ranks, in place (GradAllReduce in one part)."""
    sync = GradAllReduce(flat, 0, group)
    sync.launch()
    sync.wait()
    return flat


class GradAllReduce:
    """Sums a flat gradient buffer over the ranks in two parts.

    ``flat[:early]`` is final once the backward has recorded ``ready``; on CUDA
    its all-reduce is enqueued on a side stream that waits for that event, so it
    overlaps the rest of the backward.  ``flat[early:]`` follows once the whole
    backward has been enqueued.  ``wait()`` makes the caller's stream wait for
    both sums (call it before anything reads the gradients or the next backward
    rewrites them).  On CPU (gloo) both collectives run synchronously.  With one
    rank nothing is enqueued.  Every rank must make the same calls in the same
    order.

    The sums run in binary32 at least: a bf16 buffer is widened into a binary32
    copy, summed there and rounded back once, so each summed gradient carries
    one rounding after the ranks' own, whatever the number of ranks (a bf16 sum
    would round again at every step of the reduction).  Wider buffers are
    summed as they are.
    """

    def __init__(self, flat, early=0, group=None):
        self.flat, self.early, self.group = flat, int(early), group
        self.world = dist.get_world_size(group) if (dist.is_available() and dist.is_initialized()) else 1
        self.stream = self.ready = self.acc = None
        if self.world > 1 and torch.promote_types(flat.dtype, torch.float32) != flat.dtype:
            self.acc = torch.empty(flat.numel(), dtype=torch.float32, device=flat.device)
        if flat.is_cuda and self.world > 1:
            self.stream = torch.cuda.Stream(device=flat.device)
            if self.early > 0:
                self.ready = torch.cuda.Event()
                self.ready.record(torch.cuda.current_stream(flat.device))  # creates the CUDA event

    def ready_handle(self):
        """Raw cudaEvent_t of ``ready`` for the library to record (0 = none)."""
        return self.ready.cuda_event if self.ready is not None else 0

    def _sum(self, lo, hi):
        """All-reduce flat[lo:hi] (through the binary32 copy for a bf16 buffer)."""
        part = self.flat[lo:hi]
        if self.acc is None:
            dist.all_reduce(part, op=dist.ReduceOp.SUM, group=self.group)
            return
        acc = self.acc[lo:hi]
        acc.copy_(part)
        dist.all_reduce(acc, op=dist.ReduceOp.SUM, group=self.group)
        part.copy_(acc)

    def launch(self):
        """Enqueue the sums; call right after enqueueing the backward."""
        if self.world == 1:
            return
        n = self.flat.numel()
        if self.stream is None:
            for lo, hi in ((0, self.early), (self.early, n)):
                if hi > lo:
                    self._sum(lo, hi)
            return
        main = torch.cuda.current_stream(self.flat.device)
        with torch.cuda.stream(self.stream):
            if self.early > 0:
                self.stream.wait_event(self.ready)
                self._sum(0, self.early)
            self.stream.wait_stream(main)
            if self.early < n:
                self._sum(self.early, n)

    def wait(self):
        if self.stream is not None:
            torch.cuda.current_stream(self.flat.device).wait_stream(self.stream)


def make_step(forward, backward, sync):
    """One data-parallel training step over this rank's shard: ``forward()``,
    ``backward(ready)`` (which writes the adapter gradients into the flat
    buffer's views and records ``ready`` once the early part is final), then the
    gradient sums.  The benchmark times exactly this step; the CPU tests run it
    on gloo ranks with the oracle standing in for the kernels."""
    def step():
        forward()
        backward(sync.ready_handle())
        sync.launch()
        sync.wait()
    return step
