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
order without block resets.
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
