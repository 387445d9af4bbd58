"""Double-buffered adapter slots: the trainer's next adapter is uploaded, and its
rotations built, into the slot that compute is not using, so publishing new
adapter weights never stalls the step that is running ("Orbit", chooseai.io news
4086, section "适配器优先架构的五大设计特性": only the small BF16 adapter moves between
training and rollout, into one of two adapter slots).

Host-side orchestration over the binding: two device copies of the packed Q and
of its rotations R, a copy stream, and events that order the upload after the
last compute that read the target slot and the compute after the upload.
"""

from typing import Optional, Tuple

import torch

from .binding import oft_build_rotation


class AdapterSlots:
    """Two slots of (Q bf16 [..., b(b-1)/2], R fp32 [..., b, b]) on one device.

    upload(q) copies q (a CPU tensor; pinned for an asynchronous copy) into the
    inactive slot and builds its rotations, all on the copy stream; activate()
    makes the compute stream wait for that, marks where the compute stream stops
    reading the old slot, and returns the new slot's (Q, R)."""

    def __init__(self, q_shape: Tuple[int, ...], b: int, device, copy_stream: Optional[torch.cuda.Stream] = None):
        nq = b * (b - 1) // 2
        if q_shape[-1] != nq:
            raise ValueError(f"the last dimension of Q must be b(b-1)/2 = {nq}")
        self.b = b
        self.device = torch.device(device)
        self.q = [torch.zeros(q_shape, dtype=torch.bfloat16, device=self.device) for _ in range(2)]
        self.r = [torch.empty(*q_shape[:-1], b, b, dtype=torch.float32, device=self.device) for _ in range(2)]
        self.copy_stream = copy_stream if copy_stream is not None else torch.cuda.Stream(self.device)
        self.ready = [torch.cuda.Event() for _ in range(2)]
        self.released = [torch.cuda.Event() for _ in range(2)]
        self.active = 0
        self.pending = False
        for s in range(2):
            oft_build_rotation(self.q[s], b, R=self.r[s])
            self.ready[s].record()
            self.released[s].record()

    def current(self) -> Tuple[torch.Tensor, torch.Tensor]:
        """(Q, R) of the active slot."""
        return self.q[self.active], self.r[self.active]

    def upload(self, q_host: torch.Tensor) -> None:
        """Stage the next adapter into the inactive slot (asynchronous on the copy stream)."""
        if q_host.shape != self.q[0].shape or q_host.dtype != torch.bfloat16:
            raise ValueError("the next adapter must have the slots' shape and be bf16")
        slot = 1 - self.active
        with torch.cuda.stream(self.copy_stream):
            self.copy_stream.wait_event(self.released[slot])  # compute is done reading this slot
            self.q[slot].copy_(q_host, non_blocking=True)
            oft_build_rotation(self.q[slot], self.b, R=self.r[slot], stream=self.copy_stream)
            self.ready[slot].record(self.copy_stream)
        self.pending = True

    def activate(self, stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
        """Switch compute to the uploaded slot: `stream` (default: the current stream) waits
        for the upload, and stops reading the old slot from here on."""
        if not self.pending:
            raise RuntimeError("activate() without a preceding upload()")
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        slot = 1 - self.active
        s.wait_event(self.ready[slot])
        self.released[self.active].record(s)
        self.active = slot
        self.pending = False
        return self.current()
