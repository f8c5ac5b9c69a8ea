"""Per-step refresh of the rollout engine's FP8 weights.

"Resumen Técnico: Jet-RL", «Arquitectura Central»: the master weights stay in BF16 while
the training forward pass and the rollout both run the same FP8 linear layer, so after
every optimizer step the rollout side needs the new weights in exactly the FP8 form the
trainer's forward pass uses (128x128 blocks, «Esquema de Cuantización»), with no
calibration in between. Here the trainer quantizes each BF16 master with the library's
weight quantizer (`fp8q_quant_weight_128x128`, no transposed copy) straight into one
packed device buffer, and a single broadcast over the process group (NCCL over
NVLink / NVSwitch between GPUs) delivers every code and scale to all rollout ranks.
The rollout ranks read `qw` / `sw` as views of that buffer and pass them to
`fp8q_linear_fwd` unchanged.

One packed buffer means one collective per refresh whatever the number of weights, and
NCCL's broadcast (a pipelined ring or tree, or NVSwitch multicast where it has it)
moves each byte across each link once however many rollout ranks there are.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import quant_weight_128x128

_ALIGN = 16  # every code and scale array starts on a 16-byte boundary (TMA, vector loads)


def _align(n: int) -> int:
    return (n + _ALIGN - 1) // _ALIGN * _ALIGN


class PackedFp8Weights:
    """Codes and 128x128 scales of several weights in one contiguous uint8 buffer.

    shapes: {name: (N, K)} with N % 128 == 0 and K % 128 == 0, in a fixed order that
    every rank must share. Layout: for each weight in order, its codes [N][K] (one byte
    each) then its scales [N/128][K/128] (fp32), each array 16-byte aligned."""

    def __init__(self, shapes: dict, device):
        self.layout = {}
        off = 0
        for name, (n, k) in shapes.items():
            if n % 128 or k % 128 or n <= 0 or k <= 0:
                raise ValueError("%s: weight dimensions must be positive multiples of 128" % name)
            q_off = off
            off = _align(off + n * k)
            s_off = off
            off = _align(off + 4 * (n // 128) * (k // 128))
            self.layout[name] = (n, k, q_off, s_off)
        self.nbytes = off
        self.buffer = torch.empty(off, dtype=torch.uint8, device=device)

    def views(self) -> dict:
        """{name: (qw uint8 [N, K], sw fp32 [N/128, K/128])}, views of the buffer."""
        out = {}
        for name, (n, k, q_off, s_off) in self.layout.items():
            qw = self.buffer[q_off:q_off + n * k].view(n, k)
            sw = self.buffer[s_off:s_off + 4 * (n // 128) * (k // 128)].view(torch.float32)
            out[name] = (qw, sw.view(n // 128, k // 128))
        return out


def _quantize_into(packed: PackedFp8Weights, masters: dict, stream=None) -> None:
    views = packed.views()
    for name in packed.layout:
        qw, sw = views[name]
        quant_weight_128x128(masters[name], qw, sw, None, stream)


def refresh(packed: PackedFp8Weights, masters: dict | None = None, group=None, src: int = 0,
            quantize=None, stream=None) -> None:
    """One weight refresh. The rank `src` (a global rank) quantizes `masters` ({name: BF16
    [N, K]}) into `packed`; then, if a process group with more than one rank is active,
    `packed.buffer` is broadcast from `src` to every rank of `group`. Every rank calls
    this at the same point (a collective). `quantize(packed, masters)` replaces the
    library's quantizer (for host-side tests of the distribution alone)."""
    distributed = dist.is_available() and dist.is_initialized()
    rank = dist.get_rank() if distributed else 0
    if rank == src:
        if masters is None:
            raise ValueError("the source rank needs the BF16 master weights")
        (quantize or (lambda p, m: _quantize_into(p, m, stream)))(packed, masters)
    if distributed and dist.get_world_size(group) > 1:
        if packed.buffer.is_cuda:
            # the quantizer's kernels run on `stream`; the collective on torch's current one
            s = torch.cuda.current_stream() if stream is None else stream
            torch.cuda.current_stream().wait_stream(s)
        dist.broadcast(packed.buffer, src=src, group=group)
