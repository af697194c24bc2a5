"""Sign-Muon as deployed on the "SignMuon" summary's distributed flow: one GPU per
worker, one exchange per step.

Each rank is one worker. Per step it updates and orthogonalises its own
momentum (flow steps 1-2), turns the polar factor into signs, and the ranks
exchange them in one of the two forms of flow step 3:

* ``"allgather"``: 1 bit per parameter (entry i at bit i % 32 of word i / 32);
  every rank gathers all ranks' messages and counts the set bits (sum =
  2 * popcount - M, flow step 4). For a matrix whose column count is a
  multiple of 32 the Newton-Schulz epilogue writes the message itself (a BITS
  output) and the fused vote/update kernel reads the gathered messages: no U,
  no sign matrix and no vote matrix reach memory. Other matrices take int8
  signs from the epilogue, smuon_sign_pack and smuon_vote.
* ``"allreduce_int8"``: the +-1 signs as int8 (written by the Newton-Schulz
  epilogue), summed by an all-reduce; the vote is the sign of the sum.

Every rank then applies the same vote to its replica of W (flow step 4), so
the replicas stay identical. The exchange itself is torch.distributed (NCCL
on GPUs); the helpers below take and return plain tensors, so the host-side
logic runs on any backend. The CUDA work is the library's: smuon_ns,
smuon_sign_pack, smuon_vote and smuon_update.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (NS_FP32_REF, NS_SIMT_BF16, Bits, packed_words, smuon_ns, smuon_ns_workspace_bytes, smuon_sign_pack,
               smuon_update, smuon_vote, workspace)

EXCHANGES = ("allgather", "allreduce_int8")


def exchange_packed(packed_local: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather of the ranks' packed messages: [words] int32 in, [world, words] out in rank order."""
    world = dist.get_world_size(group)
    out = torch.empty((world, packed_local.numel()), dtype=packed_local.dtype, device=packed_local.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, packed_local.contiguous(), group=group)
    else:
        dist.all_gather(list(out.unbind(0)), packed_local.contiguous(), group=group)
    return out


def exchange_signs_int8(signs_local: torch.Tensor, group=None) -> torch.Tensor:
    """All-reduce (sum) of the ranks' +-1 int8 signs; |sum| <= world, so int8 holds it for up to 127 ranks."""
    if dist.get_world_size(group) > 127:
        raise ValueError("the int8 sum holds at most 127 workers")
    out = signs_local.contiguous().clone()
    dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
    return out


def payload_bytes(n_params: int, world: int, exchange: str) -> dict:
    """Bytes one rank sends per step for n_params parameters (SignMuon summary,
    communication efficiency): its 1-bit message (n/8, 32x less than float32)
    or its int8 signs (n, 4x less), against a float32 exchange of the same
    parameters (4n)."""
    sent = n_params / 8 if exchange == "allgather" else n_params
    return {"sent": sent, "f32": 4 * n_params, "ratio_vs_f32": 4 * n_params / sent, "world": world}


class DistributedSignMuon:
    """One worker of Sign-Muon per rank. ``W`` (replicated on every rank) and the
    rank's own momentum ``M`` are lists of 2-D CUDA tensors of the same shapes;
    ``step(G)`` takes this rank's gradients."""

    def __init__(self, W, M, coeffs, iters, beta, eta, exchange="allgather", tie_value=0, ns_flags=0,
                 group=None):
        if exchange not in EXCHANGES:
            raise ValueError(f"exchange must be one of {EXCHANGES}")
        self.W, self.M = list(W), list(M)
        self.coeffs, self.iters, self.beta, self.eta = coeffs, iters, beta, eta
        self.exchange, self.tie, self.flags, self.group = exchange, tie_value, ns_flags, group
        self.world = dist.get_world_size(group)
        dev = self.W[0].device
        tensor_cores = not (ns_flags & (NS_FP32_REF | NS_SIMT_BF16))
        # matrices whose message the Newton-Schulz epilogue writes directly
        self.bits = [exchange == "allgather" and tensor_cores and w.shape[1] % 32 == 0 for w in self.W]
        self.U = [Bits.empty(*w.shape, device=dev) if b else torch.empty(w.shape, dtype=torch.int8, device=dev)
                  for w, b in zip(self.W, self.bits)]
        self.votes = [torch.empty(w.numel(), dtype=torch.int8, device=dev) for w in self.W]
        self.ws = workspace(smuon_ns_workspace_bytes(self.M, iters, ns_flags), dev)
        if exchange == "allgather":
            self.local = [u.words if b else torch.empty(packed_words(w.numel()), dtype=torch.int32, device=dev)
                          for u, w, b in zip(self.U, self.W, self.bits)]
        else:
            self.local = [u.view(1, -1) for u in self.U]

    def payload(self) -> dict:
        return payload_bytes(sum(w.numel() for w in self.W), self.world, self.exchange)

    def step(self, G):
        # flow steps 1-2: momentum and polar factor of this worker (its signs or message only)
        smuon_ns(self.M, self.U, *self.coeffs, self.iters, G=list(G), beta=self.beta, flags=self.flags, ws=self.ws)
        msgs, voted = [], []
        for l, w in enumerate(self.W):
            n = w.numel()
            if self.exchange == "allgather":
                if not self.bits[l]:
                    smuon_sign_pack([self.U[l]], packed=self.local[l].view(1, -1))
                gathered = exchange_packed(self.local[l], self.group)
                if self.bits[l]:
                    msgs.append((l, [Bits(gathered[k], *w.shape) for k in range(self.world)]))
                    continue
                smuon_vote(self.world, n, self.votes[l], packed=gathered, tie_value=self.tie)
            else:  # the int8 signs came straight from the Newton-Schulz epilogue
                total = exchange_signs_int8(self.local[l], self.group)
                smuon_vote(1, n, self.votes[l], signs_i8=total, tie_value=self.tie)  # sign of the summed signs
            voted.append(l)
        # flow step 4: the same update on every replica -- the gathered messages straight into the fused
        # vote / update kernel, the other matrices from their votes
        if msgs:
            smuon_update([self.W[l] for l, _ in msgs], self.eta, U=[m for _, m in msgs], M=self.world,
                         tie_value=self.tie)
        if voted:
            smuon_update([self.W[l] for l in voted], self.eta,
                         votes=[self.votes[l].view(self.W[l].shape) for l in voted])
