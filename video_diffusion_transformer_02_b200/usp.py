"""Unified sequence parallelism for the spatiotemporal attention of a DiT
layer across GPUs (ReGenVC "Unified sequence parallelism", Sec. 3.5:
DeepSpeed-Ulysses all-to-all over U ranks composed with Ring attention over
R ranks, U x R ranks in all, exact up to reduction order).

Every rank starts with a contiguous slice of the token sequence, [B, L/(U R),
H, d], of q, k and v.
  * Ulysses (a group of U ranks): an all-to-all turns the group's U token
    slices into whole-group sequences of H/U heads each, [B, L/R, H/U, d];
    the inverse all-to-all turns the attention output back into token
    slices.
  * Ring (a group of R ranks): each rank attends its query slice to the
    key/value slice it holds and passes that slice on to the next rank, R
    times; the R partial attentions are joined exactly through their
    log-sum-exp.
The data plane is torch.distributed (NCCL over NVLink on GPUs; point-to-point
sends for the ring, all_to_all_single for Ulysses; no multicast).  The
attention of one shard and the join are callables: on the GPU the library's
vattn_attention (with its lse output) and vattn_attention_merge
(gpu_attend / gpu_merge below); any other pair with the same contract can be
passed, e.g. to check the partition arithmetic.

Contract of attend(q, k, v, q_tok0, k_tok0) -> (o, lse): q [B, Lq, h, d] at
global token positions q_tok0.., k/v [B, Lk, hkv, d] at k_tok0..; o [B, Lq,
h, d], lse [B, h, Lq] (natural log of the softmax denominator, -inf where no
key of the shard is visible).  merge(o_parts [R, B, Lq, h, d], lse_parts
[R, B, h, Lq]) -> o [B, Lq, h, d].
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def _group_size(group):
    return dist.get_world_size(group)


def _bytes(t: torch.Tensor) -> torch.Tensor:
    # the wires carry raw bytes: every backend moves uint8, and the values
    # arrive bit for bit whatever their type
    return t.view(torch.uint8)


def ulysses_tokens_to_heads(x: torch.Tensor, group) -> torch.Tensor:
    """[B, Ls, H, d] token slice of this rank -> [B, U * Ls, H / U, d]: the
    whole group's tokens (rank u's slice at u * Ls) for head group `rank`."""
    U = _group_size(group)
    if U == 1:
        return x
    B, Ls, H, d = x.shape
    if H % U:
        raise ValueError("heads (%d) must divide by the Ulysses group size (%d)" % (H, U))
    send = x.reshape(B, Ls, U, H // U, d).permute(2, 0, 1, 3, 4).contiguous()   # [U, B, Ls, H/U, d]
    recv = torch.empty_like(send)
    dist.all_to_all_single(_bytes(recv), _bytes(send), group=group)   # chunk u: rank u's tokens, my heads
    return recv.permute(1, 0, 2, 3, 4).reshape(B, U * Ls, H // U, d).contiguous()


def ulysses_heads_to_tokens(y: torch.Tensor, group) -> torch.Tensor:
    """Inverse of ulysses_tokens_to_heads: [B, U * Ls, H / U, d] -> [B, Ls, H, d]."""
    U = _group_size(group)
    if U == 1:
        return y
    B, L, Hu, d = y.shape
    Ls = L // U
    send = y.reshape(B, U, Ls, Hu, d).permute(1, 0, 2, 3, 4).contiguous()       # chunk u: rank u's tokens
    recv = torch.empty_like(send)
    dist.all_to_all_single(_bytes(recv), _bytes(send), group=group)   # chunk u: my tokens, head group u
    return recv.permute(1, 2, 0, 3, 4).reshape(B, Ls, U * Hu, d).contiguous()


def ring_attention(q, k, v, group, attend, merge, q_tok0: int, kv_len: int):
    """Ring attention over the R ranks of `group`: rank r holds key/value
    slice r (tokens [r * kv_len, (r + 1) * kv_len)); after R steps every rank
    has attended its queries (at q_tok0..) to all slices, which are joined by
    `merge`."""
    R = _group_size(group)
    r = dist.get_rank(group)
    nxt = dist.get_global_rank(group, (r + 1) % R)
    prv = dist.get_global_rank(group, (r - 1) % R)
    o_parts, lse_parts = [], []
    kc, vc = k.contiguous(), v.contiguous()
    for i in range(R):
        j = (r - i) % R                                       # the slice held at step i
        if i + 1 < R:                                         # pass it on while attending to it
            kn, vn = torch.empty_like(kc), torch.empty_like(vc)
            reqs = dist.batch_isend_irecv([dist.P2POp(dist.isend, _bytes(kc), nxt, group),
                                           dist.P2POp(dist.isend, _bytes(vc), nxt, group),
                                           dist.P2POp(dist.irecv, _bytes(kn), prv, group),
                                           dist.P2POp(dist.irecv, _bytes(vn), prv, group)])
        o, lse = attend(q, kc, vc, q_tok0, j * kv_len)
        o_parts.append(o)
        lse_parts.append(lse)
        if i + 1 < R:
            for rq in reqs:
                rq.wait()
            kc, vc = kn, vn
    if R == 1:
        return o_parts[0]
    return merge(torch.stack(o_parts), torch.stack(lse_parts))


def usp_attention(q, k, v, ulysses_group, ring_group, attend, merge, tok0: int):
    """Attention of the whole sequence, computed by U x R ranks.

    q/k/v: this rank's token slice [B, Ls, H, d] (k/v with Hkv heads), at
    global tokens tok0..tok0+Ls; the ranks of a Ulysses group hold
    consecutive slices, and Ulysses group g of the ring is sequence block g.
    Returns this rank's slice of the output, [B, Ls, H, d]."""
    U = _group_size(ulysses_group)
    Ls = q.shape[1]
    u = dist.get_rank(ulysses_group)
    qh = ulysses_tokens_to_heads(q, ulysses_group)
    kh = ulysses_tokens_to_heads(k, ulysses_group)
    vh = ulysses_tokens_to_heads(v, ulysses_group)
    block0 = tok0 - u * Ls                                    # first token of the Ulysses group's block
    oh = ring_attention(qh, kh, vh, ring_group, attend, merge, block0, U * Ls)
    return ulysses_heads_to_tokens(oh, ulysses_group)


# --------------------------------------------------- the library's kernels
def gpu_attend(scale, mode="full", tokens_per_frame=0, chunk_frames=1, window_back=0, window_fwd=0, rope=None,
               table=None):
    """attend() through vattn_attention: frame offsets from the token
    offsets (slices must start on frame boundaries when masks or RoPE are
    used)."""
    from . import vattn_attention

    def attend(q, k, v, q_tok0, k_tok0):
        F = tokens_per_frame if tokens_per_frame else 1
        if (mode != "full" or rope is not None) and (q_tok0 % F or k_tok0 % F):
            raise ValueError("slices must start on frame boundaries")
        B, Lq, H, d = q.shape
        o = torch.empty_like(q)
        lse = torch.empty((B, H, Lq), dtype=torch.float32, device=q.device)
        vattn_attention(q, k, v, o, lse, scale=scale, mode=mode, tokens_per_frame=tokens_per_frame,
                        chunk_frames=chunk_frames, window_back=window_back, window_fwd=window_fwd,
                        q_frame_offset=q_tok0 // F, k_frame_offset=k_tok0 // F, rope=rope, table=table)
        return o, lse
    return attend


def gpu_merge(o_parts, lse_parts):
    """merge() through vattn_attention_merge."""
    from . import vattn_attention_merge
    o = torch.empty(o_parts.shape[1:], dtype=o_parts.dtype, device=o_parts.device)
    vattn_attention_merge(o_parts.contiguous(), lse_parts.contiguous(), o)
    return o
