"""The forward scan split along the sequence across ranks (host-side exchange).

Rank r holds tokens [t_r, t_{r+1}) of every sequence (the same batch rows and
heads on every rank).  The chunked algorithm's state hand-off, one level up
(d-central.tech glossary "State Space Duality": attention-like blocks, a
recurrence between them; aifetchly blog "Mamba-2 Architecture", "The Chunked
SSD Algorithm", step 2):

1. local pass: S_r = the state the slice alone leaves (scan from state 0),
   and alpha_r [B, H], the slice's total decay exp(sum_t dt_t A_h), read off a
   scan of x = 0 from an all-ones state;
2. one all-gather of (alpha_q, S_q) over the ranks;
3. s_in_r = sum_{q < r} (prod_{q < q' < r} alpha_q') S_q
            + (prod_{q < r} alpha_q) h0                         (h0: the global
   initial state, known to every rank), i.e. the state-passing recurrence
   s_in_{q+1} = alpha_q s_in_q + S_q over the ranks;
4. the slice again from s_in_r: its y and its final state are then exact.

`local_scan(x, dt, A, B, C, D, chunk_len, h0) -> (y, final)` is the per-rank
scan: the library's ``binding.forward`` on a GPU.  Everything here is argument
handling and the exchange; the per-token arithmetic is the local scan's.
"""
from __future__ import annotations

import torch


def slice_summary(local_scan, x, dt, A, B, C, chunk_len=256):
    """Step 1 for one slice: (alpha [B, H], S [B, H, P, N]).

    S is the state the slice leaves when it starts from zero; alpha is the
    slice's total decay, read off a scan of x = 0 from an all-ones state (the
    states keep the local scan's dtype: fp32 from the library, fp64 from a
    reference scan).
    """
    bsz, _, H, P = x.shape
    N = B.shape[3]
    _, S = local_scan(x, dt, A, B, C, None, chunk_len, None)
    ones = torch.ones((bsz, H, P, N), dtype=S.dtype, device=x.device)
    _, decayed = local_scan(torch.zeros_like(x), dt, A, B, C, None, chunk_len, ones)
    return decayed[:, :, 0, 0].contiguous(), S


def entering_state(alphas, states, rank, h0=None):
    """Step 3: the state entering slice `rank` from the summaries of the slices
    before it (lists indexed by rank) and the whole sequence's initial state."""
    S0 = states[0]
    s_in = h0.to(S0.dtype).clone() if h0 is not None else torch.zeros_like(S0)
    for q in range(rank):
        s_in = alphas[q][:, :, None, None] * s_in + states[q]
    return s_in


def forward_sequence_split(local_scan, x, dt, A, B, C, D=None, chunk_len=256, h0=None, group=None):
    """Sequence-parallel forward scan of this rank's slice.

    x [B, T_r, H, P], dt [B, T_r, H], B/C [B, T_r, G, N]: this rank's tokens;
    A, D [H]; h0 [B, H, P, N] (the initial state of the whole sequence, or
    None).  Returns (y [B, T_r, H, P], final [B, H, P, N]) where final is the
    state after this rank's last token.  Collective: every rank of `group`
    calls it once with slices in rank order.
    """
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    bsz, _, H, P = x.shape
    N = B.shape[3]
    # 1. the state the slice alone leaves, and its total decay
    alpha, S = slice_summary(local_scan, x, dt, A, B, C, chunk_len)
    # 2. one all-gather of (alpha, S)
    payload = torch.cat([alpha.reshape(-1), S.reshape(-1)])
    gathered = [torch.empty_like(payload) for _ in range(world)]
    dist.all_gather(gathered, payload, group=group)
    na = alpha.numel()
    alphas = [g[:na].reshape(bsz, H) for g in gathered]
    states = [g[na:].reshape(bsz, H, P, N) for g in gathered]
    # 3. the state entering this rank: the recurrence over the ranks before it
    s_in = entering_state(alphas, states, rank, h0)
    # 4. the slice from its true incoming state
    return local_scan(x, dt, A, B, C, D, chunk_len, s_in)
