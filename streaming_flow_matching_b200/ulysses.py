"""Ulysses context parallelism of the performer: the host-side data movement.

The performer runs as a multi-GPU group with Ulysses-style context parallelism:
the long video latent sequence is split along the token axis across the P
ranks, an all-to-all before each attention turns token shards into head
shards (every rank then holds the whole sequence for H / P heads) and another
one turns them back; audio latents are short and are not sharded (every rank
computes the whole audio part); the ranks gather the unit's latents at the end;
each rank's K/V cache is pre-sharded, so the thinker's broadcast slice is
appended per rank without a collective ("Wan-Streamer v0.2: Higher Resolution,
Same Latency" digest, "method overview and architecture"; "Wan-Streamer v0.2"
blog, "Infra"; v0.2 abstract).

This module holds only the index maps and the exchanges, no arithmetic of the
method: which tokens and heads each rank owns, how the buffers of the two
all-to-alls are laid out, and the exchanges themselves through
``torch.distributed`` (NCCL between GPUs, gloo on CPU).  The kernels of a rank
(projections, attention over its head group, head and Euler update) are the
single-GPU ones applied to that rank's rows and heads.

Layouts (P ranks, Nv video and Na audio tokens, H heads of D dims):
  * video shard of rank r: tokens [r Nv / P, (r + 1) Nv / P) (floor division;
    contiguous, the last shards may differ by one token);
  * head group of rank r: heads [r H / P, (r + 1) H / P) (H divisible by P);
  * local rows of rank r: its video shard, then all Na audio tokens -- the unit's
    own order (video, then audio) restricted to the rank's tokens;
  * sequence -> heads: rank r sends rows [0, nv_r) x heads of rank s to rank s;
    the received blocks, in rank order, are the unit's video tokens in order;
    the audio rows of its own heads follow from its local rows;
  * heads -> sequence: rank r sends the video rows of rank s's shard (its heads)
    to rank s; audio rows of every head group are all-gathered.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass(frozen=True)
class UlyssesPlan:
    """Token and head ownership of a P-rank Ulysses group."""
    n_video: int
    n_audio: int
    n_heads: int
    world: int

    def __post_init__(self):
        if self.world < 1 or self.n_heads % self.world:
            raise ValueError("the head count must be a multiple of the group size")
        if self.n_video < self.world:
            raise ValueError("every rank needs at least one video token")

    @property
    def n_tokens(self):
        return self.n_video + self.n_audio

    @property
    def heads_per_rank(self):
        return self.n_heads // self.world

    def video_range(self, r):
        """[start, end) of rank r's video tokens."""
        return r * self.n_video // self.world, (r + 1) * self.n_video // self.world

    def n_video_local(self, r):
        a, b = self.video_range(r)
        return b - a

    def n_local(self, r):
        return self.n_video_local(r) + self.n_audio

    def head_range(self, r):
        """[start, end) of rank r's heads (its share of a head-sharded cache)."""
        return r * self.heads_per_rank, (r + 1) * self.heads_per_rank

    def local_tokens(self, r):
        """Unit token indices of rank r's local rows: its video shard, then the audio."""
        a, b = self.video_range(r)
        return list(range(a, b)) + list(range(self.n_video, self.n_tokens))


def _group_size(group):
    return dist.get_world_size(group)


def seq_to_heads(plan: UlyssesPlan, x_local, rank, group=None):
    """All-to-all before attention: [n_local(rank)][H][D] -> [N][H/P][D].

    Rows of the result follow the unit's order: every video token (gathered
    from the ranks' shards, in rank order), then the audio tokens, for this
    rank's head group.  Audio rows come from the local copy (replicated)."""
    P, hp = plan.world, plan.heads_per_rank
    assert _group_size(group) == P
    nv = plan.n_video_local(rank)
    D = x_local.shape[-1]
    # send block s: my video rows, heads of rank s -> contiguous
    send = torch.cat([x_local[:nv, s * hp:(s + 1) * hp].reshape(-1) for s in range(P)])
    in_splits = [nv * hp * D] * P
    out_splits = [plan.n_video_local(s) * hp * D for s in range(P)]
    recv = torch.empty(sum(out_splits), dtype=x_local.dtype, device=x_local.device)
    dist.all_to_all_single(recv, send, out_splits, in_splits, group=group)
    h0, h1 = plan.head_range(rank)
    video = recv.view(plan.n_video, hp, D)
    audio = x_local[nv:, h0:h1]
    return torch.cat([video, audio], dim=0)


def heads_to_seq(plan: UlyssesPlan, o_heads, rank, group=None):
    """All-to-all after attention: [N][H/P][D] (this rank's heads) -> [n_local][H][D].

    Video rows go back to the rank owning the token; the audio rows of every
    head group are all-gathered (every rank keeps the whole audio part)."""
    P, hp = plan.world, plan.heads_per_rank
    assert _group_size(group) == P
    D = o_heads.shape[-1]
    nv = plan.n_video_local(rank)
    send = o_heads[:plan.n_video].reshape(-1).contiguous()
    in_splits = [plan.n_video_local(s) * hp * D for s in range(P)]
    out_splits = [nv * hp * D] * P
    recv = torch.empty(sum(out_splits), dtype=o_heads.dtype, device=o_heads.device)
    dist.all_to_all_single(recv, send, out_splits, in_splits, group=group)
    out = torch.empty(plan.n_local(rank), plan.n_heads, D, dtype=o_heads.dtype,
                      device=o_heads.device)
    blocks = recv.view(P, nv, hp, D)
    for s in range(P):
        out[:nv, s * hp:(s + 1) * hp] = blocks[s]
    audio = [torch.empty_like(o_heads[plan.n_video:]) for _ in range(P)]
    dist.all_gather(audio, o_heads[plan.n_video:].contiguous(), group=group)
    for s in range(P):
        out[nv:, s * hp:(s + 1) * hp] = audio[s]
    return out


def gather_latents(plan: UlyssesPlan, z_local, rank, group=None):
    """The unit's latents [N][C] on every rank from each rank's local rows [n_local][C]
    (video shards gathered in rank order, audio from the local copy)."""
    P = plan.world
    assert _group_size(group) == P
    nv = plan.n_video_local(rank)
    width = max(plan.n_video_local(s) for s in range(P))
    pad = torch.zeros(width, *z_local.shape[1:], dtype=z_local.dtype, device=z_local.device)
    pad[:nv] = z_local[:nv]
    parts = [torch.empty_like(pad) for _ in range(P)]
    dist.all_gather(parts, pad, group=group)
    video = torch.cat([parts[s][:plan.n_video_local(s)] for s in range(P)], dim=0)
    return torch.cat([video, z_local[nv:]], dim=0)


def cache_heads(plan: UlyssesPlan, k_slice, rank):
    """Rank r's share of a broadcast K/V slice [..][H][D]: heads of its group (what
    sfm_kvcache_append_heads copies on the GPU)."""
    h0, h1 = plan.head_range(rank)
    return k_slice[..., h0:h1, :]
