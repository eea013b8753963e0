"""Classifier-free guidance split over two GPUs.

The sampling loop's CFG batch is [uncond; text] ("在 AuraFlowPipeline 中的实际
调用" in the architecture guide: the latents are duplicated, the velocity is
chunked into the uncond and text halves, uncond first; the guidance formula
is in the pipeline guide's parameter section).  The two halves are
independent forwards, so one process per GPU takes one half: rank 0 the
unconditional prompt, rank 1 the text prompt.  Per step each rank runs the
forward on its Bi samples and both ranks apply the same guidance + Euler
update, so their latents stay identical without any further exchange.  Two
ways to bring the other half in:

* ``exchange="peer"`` (the fused form): each rank writes its half into one
  of two slots of an exchange buffer that the other rank maps through CUDA
  IPC (handles sent with one ``all_gather_object`` at set-up); after the
  forward, a stream sync and one host barrier, the guidance + Euler kernel
  reads the local half and the peer's half straight from the peer GPU's
  memory.  Slots alternate per step, so a slot is rewritten only after the
  peer has passed the next barrier, i.e. finished reading it.
* ``exchange="nccl"``: one NCCL all-gather of the two [Bi, C, H, W] halves
  (rank order = uncond first) into a local [2 Bi, ...] buffer, then the
  guidance + Euler kernel on it.

Every compute step runs in this package's CUDA library; torch.distributed
carries the set-up exchange, the barrier or the collective.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import Exchange, euler_cfg_step, euler_cfg_step2, transformer_forward


class CFGSplitSampler:
    """One rank of a 2-rank CFG split.

    latents:  [Bi, C, H, W] float32 (updated in place, identical on both ranks)
    text_emb: [2 Bi, L, joint_attention_dim] bf16, uncond rows first; this
              rank keeps rows [rank Bi, (rank + 1) Bi)
    sigmas:   n_steps + 1 floats
    text_len: optional int32 [2 Bi] real prompt lengths (padded prompts)
    exchange: "peer" (fused peer-memory exchange) or "nccl" (all-gather)
    """

    def __init__(self, w, s, latents, text_emb, sigmas, guidance: float, group=None, text_len=None,
                 exchange: str = "peer", _forward=None, _euler=None, _euler2=None, _make_exchange=None):
        world = dist.get_world_size(group)
        if world != 2:
            raise ValueError(f"the CFG split needs exactly 2 ranks, the group has {world}")
        if exchange not in ("peer", "nccl"):
            raise ValueError(f"exchange must be 'peer' or 'nccl', got {exchange!r}")
        self.rank = dist.get_rank(group)
        Bi = latents.shape[0]
        if text_emb.shape[0] != 2 * Bi:
            raise ValueError("text_emb must hold 2*Bi rows (uncond first)")
        self.group = group
        self.exchange = exchange
        self.latents = latents
        self.sigmas = [float(x) for x in sigmas]
        self.guidance = float(guidance)
        r0 = self.rank * Bi
        self.text_half = text_emb[r0:r0 + Bi].contiguous()
        self.text_len = None if text_len is None else text_len[r0:r0 + Bi].contiguous()
        dev = latents.device
        # model time of every step for this rank's samples, one upload
        self.t = torch.tensor([[sg] * Bi for sg in self.sigmas[:-1]], dtype=latents.dtype).to(dev)
        # everything runs on the current CUDA stream, which the collective also orders against
        self._forward = _forward or (lambda lat, txt, t, vel, tl: transformer_forward(
            w, s, lat, txt, t, vel, text_len=tl))
        if exchange == "nccl":
            self.vel_half = torch.empty_like(latents)
            self.vel_pair = torch.empty((2 * Bi,) + tuple(latents.shape[1:]), dtype=latents.dtype, device=dev)
            self._euler = _euler or (lambda lat, v, g, a, b: euler_cfg_step(lat, v, g, a, b))
        else:
            self._ex = (_make_exchange or (lambda shape: Exchange(shape, slots=2)))(tuple(latents.shape))
            handles = [None, None]
            dist.all_gather_object(handles, self._ex.handle(), group=group)
            self._ex.open_peer(handles[1 - self.rank])
            self._euler2 = _euler2 or (lambda lat, vu, vc, g, a, b: euler_cfg_step2(lat, vu, vc, g, a, b))

    @property
    def n_steps(self) -> int:
        return len(self.sigmas) - 1

    def step(self, i: int):
        if not 0 <= i < self.n_steps:
            raise IndexError(f"step {i} outside [0, {self.n_steps})")
        if self.exchange == "nccl":
            self._forward(self.latents, self.text_half, self.t[i], self.vel_half, self.text_len)
            dist.all_gather_into_tensor(self.vel_pair, self.vel_half, group=self.group)   # [uncond; text]
            self._euler(self.latents, self.vel_pair, self.guidance, self.sigmas[i], self.sigmas[i + 1])
            return
        slot = i % 2
        mine = self._ex.local(slot)
        self._forward(self.latents, self.text_half, self.t[i], mine, self.text_len)
        self._ex.synchronize()              # this rank's half of step i is complete
        dist.barrier(group=self.group)      # and so is the peer's
        theirs = self._ex.peer(slot)
        vu, vc = (mine, theirs) if self.rank == 0 else (theirs, mine)
        self._euler2(self.latents, vu, vc, self.guidance, self.sigmas[i], self.sigmas[i + 1])

    def close(self):
        ex = getattr(self, "_ex", None)
        if ex is not None:
            ex.close()
            self._ex = None
