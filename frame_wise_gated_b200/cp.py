"""Time-sharded context parallelism of the frame scan, one process per GPU.

The SANA-WM blog (blog.hotdry.top, section 显存分片：Context-Parallel 的工程实现)
splits the frames of a sequence across devices and carries the recurrence
across the split exactly: a span of frames maps its start state to its end
state affinely, S_end = S_start C_p + H_p. Here rank r of R holds frames
[r*T, (r+1)*T) of every head (rank order = time order) and:

  1. computes its span's map per head with the library's kernels
     (gdn_cp_shard_composite: C = g (I - E), H);
  2. exchanges the maps with one all-gather over the process group (NCCL on
     GPUs: 2 D^2 + 1 fp32 values per head per rank, 128 KiB per head at D=128);
  3. folds state_in through the maps of ranks 0..r-1 (gdn_cp_prefix) into its
     exact start state;
  4. scans its own frames from that state (gdn_frame_scan_fwd_ex).

Every rank takes the same collective steps in the same order. Forward scan
order without block resets (frame_scan_fwd_cp), or the bidirectional
chunk-causal form (frame_scan_bidir_cp): the forward direction as above, and
the reverse direction, which restarts at every block of `block` frames, runs
on each rank alone when the shards hold whole blocks.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from frame_wise_gated_b200 import api


class KernelBackend:
    """The library's CUDA kernels (the product path)."""

    def shard_composite(self, k, v, beta, gamma):
        return api.cp_shard_composite(k, v, beta, gamma)

    def prefix(self, E_all, H_all, g_all, state_in, r):
        return api.cp_prefix(E_all, H_all, g_all, state_in, r)

    def scan(self, q, k, v, beta, gamma, state_in, **kw):
        return api.frame_scan_fwd_ex(q, k, v, beta, gamma, state_in, **kw)


def _gather(x, group):
    """All ranks' x stacked in rank order: [R, *x.shape]."""
    world = dist.get_world_size(group)
    out = torch.empty((world * x.shape[0],) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
    dist.all_gather_into_tensor(out, x.contiguous(), group=group)
    return out.view((world,) + tuple(x.shape))


def frame_scan_fwd_cp(q, k, v, beta, gamma, state_in=None, *, group=None, backend=None,
                      **scan_kw):
    """The frame scan of a sequence whose frames are split across the ranks of
    `group` in rank order. q, k, v [B,H,T,S,D], beta [B,H,T,S], gamma [B,H,T]
    hold this rank's T frames; state_in [B,H,D,D] (or None) is the state
    entering the sequence, the same on every rank. Returns this rank's
    (out, state_out); the last rank's state_out is the sequence's."""
    be = backend or KernelBackend()
    r = dist.get_rank(group)
    E, H, g = be.shard_composite(k, v, beta, gamma)
    E_all, H_all, g_all = _gather(E, group), _gather(H, group), _gather(g, group)
    s0 = be.prefix(E_all, H_all, g_all, state_in, r)
    return be.scan(q, k, v, beta, gamma, s0, **scan_kw)


def frame_scan_bidir_cp(q, k, v, beta, gamma, state_in=None, *, block=3, state_in_rev=...,
                        group=None, backend=None, **scan_kw):
    """The bidirectional chunk-causal form (forward scan without resets plus a
    reverse-time scan restarted at every block of `block` frames; SANA-WM's
    inference variant, hyper.ai summary, section 方法) of a sequence whose
    frames are split across the ranks of `group` in rank order.

    The forward direction crosses the shard boundaries exactly through the
    span maps, as in frame_scan_fwd_cp. Blocks are floor(t / block) counted
    from the sequence's first frame, so when every shard holds whole blocks
    (this rank's T a multiple of `block`, the same T on every rank) no reverse
    block spans two ranks and the reverse needs no exchange: only the block
    that comes first in reverse order (the last block, on the last rank)
    starts from a given state -- state_in_rev if passed (a tensor, or None for
    zeros), else state_in -- and every other block from zeros.

    Returns this rank's (out, state_out, out_rev, state_out_rev); the last
    rank's state_out is the sequence's forward end state, rank 0's
    state_out_rev the reverse scan's (the state after frame 0)."""
    T = q.shape[2]
    if block < 1 or T % block:
        raise ValueError(f"each rank's {T} frames must hold whole blocks of {block}")
    be = backend or KernelBackend()
    r, world = dist.get_rank(group), dist.get_world_size(group)
    E, H, g = be.shard_composite(k, v, beta, gamma)
    E_all, H_all, g_all = _gather(E, group), _gather(H, group), _gather(g, group)
    s0 = be.prefix(E_all, H_all, g_all, state_in, r)
    seed = (state_in if state_in_rev is ... else state_in_rev) if r == world - 1 else None
    return be.scan(q, k, v, beta, gamma, s0, bidir=True, block_reset=True, block=block,
                   state_in_rev=seed, **scan_kw)
