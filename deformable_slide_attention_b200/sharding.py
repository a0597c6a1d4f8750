"""Head-sharded 3D-DSA over several GPUs, one process per GPU.

3D Deformable Slide Attention (MegaSlide-DiT, arXiv 2607.22696, Eq. 1) is computed per attention
head: the operator needs every token of a head, and nothing of the other heads.  Heads therefore
split over ranks with no exchange inside the operator.  A caller whose activations are sharded by
tokens (rank r holds tokens [n_r0, n_r1) of every head, the layout of sequence-parallel training)
needs one all-to-all before the operator, to give each rank every token of its heads
[h_r0, h_r1), and one after it, to return the results to the token shards.

HeadShardedDSA does exactly that around the library's forward and backward:

    forward:  q, k, v [N_r][H][dh], offsets [H][N_r][3] (or [H][N_r][K][3])
              --all-to-all--> [N][H_r][dh], [H_r][N][3] --dsa3d_forward--> out [N][H_r][dh],
              lse [H_r][N] --all-to-all--> out [N_r][H][dh], lse [H][N_r]
    backward: dO [N_r][H][dh] --all-to-all--> [N][H_r][dh] --dsa3d_backward (on the forward's
              head shards)--> dq, dk, dv, doffsets --all-to-all--> token shards

Token ranges and head ranges are contiguous, with sizes that differ by at most one
(ranks.head_range).  The exchanges move raw bytes (torch.distributed.all_to_all_single on a
uint8 view), so they are exact for every dtype and work on NCCL and gloo alike.  The per-rank
operator calls are injectable: by default the library's (per-token or per-tap) entry points on
the rank's CUDA device; the tests on CPU pass stand-ins.  No TMA load with cluster multicast is
involved: the exchanges are NCCL's.
"""
from __future__ import annotations

from . import ranks


def token_range(N: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous tokens [n0, n1) of rank `rank` (sizes differ by at most one)."""
    return ranks.head_range(N, rank, world)


def _sizes(total, world):
    return [b - a for a, b in (ranks.head_range(total, r, world) for r in range(world))]


def _a2a_bytes(chunks, recv_bytes, group):
    """Send chunks[j] (contiguous tensors) to rank j; receive recv_bytes[i] bytes from rank i.
    Returns the received byte buffers, in rank order."""
    import torch
    import torch.distributed as dist
    send = [c.contiguous().view(-1).view(torch.uint8) for c in chunks]
    inp = torch.cat(send) if send else torch.empty(0, dtype=torch.uint8)
    out = torch.empty(sum(recv_bytes), dtype=torch.uint8, device=inp.device)
    dist.all_to_all_single(out, inp, output_split_sizes=list(recv_bytes),
                           input_split_sizes=[s.numel() for s in send], group=group)
    return list(torch.split(out, list(recv_bytes)))


class HeadShardedDSA:
    """3D-DSA on token-sharded activations, computed head-sharded (see the module docstring).

    dims = (F, Hp, Wp) of the whole clip, N = F Hp Wp; heads = H of the whole layer.  Rank r holds
    tokens token_range(N, r, world) and computes heads ranks.head_range(H, r, world).
    forward_fn(q, k, v, offsets, dims, window) -> (out, lse) and
    backward_fn(q, k, v, offsets, lse, dout, dims, window) -> (dq, dk, dv, doffsets) are the
    per-rank operator calls on head-sharded tensors (default: the library's entry points).
    """

    def __init__(self, dims, window, heads, group=None, per_tap=False, forward_fn=None,
                 backward_fn=None):
        import torch.distributed as dist
        self.dims, self.window, self.heads = tuple(dims), tuple(window), heads
        self.N = dims[0] * dims[1] * dims[2]
        self.K = window[0] * window[1] * window[2]
        self.per_tap = per_tap
        self.group = group
        on = dist.is_available() and dist.is_initialized()
        self.world = dist.get_world_size(group) if on else 1
        self.rank = dist.get_rank(group) if on else 0
        if heads < self.world or self.N < self.world:
            raise ValueError("every rank needs at least one head and one token")
        self.tokens = _sizes(self.N, self.world)
        self.head_counts = _sizes(heads, self.world)
        self.n0, self.n1 = token_range(self.N, self.rank, self.world)
        self.h0, self.h1 = ranks.head_range(heads, self.rank, self.world)
        if forward_fn is None or backward_fn is None:
            from . import abi
            fwd, bwd = (abi.forward_taps, abi.backward_taps) if per_tap else (abi.forward, abi.backward)
            forward_fn = forward_fn or fwd
            backward_fn = backward_fn or bwd
        self.forward_fn, self.backward_fn = forward_fn, backward_fn

    # --- layouts ------------------------------------------------------------------------------
    def rows_to_heads(self, x):
        """[N_r][H][...] token shard -> [N][H_r][...] head shard."""
        if self.world == 1:
            return x
        tail = tuple(x.shape[2:])
        per = x.element_size() * (1 if not tail else _prod(tail))
        chunks, h = [], 0
        for c in self.head_counts:
            chunks.append(x[:, h:h + c])
            h += c
        hr = self.h1 - self.h0
        got = _a2a_bytes(chunks, [n * hr * per for n in self.tokens], self.group)
        return _cat([g.view(x.dtype).view(n, hr, *tail) for g, n in zip(got, self.tokens)], 0)

    def rows_to_tokens(self, y):
        """[N][H_r][...] head shard -> [N_r][H][...] token shard."""
        if self.world == 1:
            return y
        tail = tuple(y.shape[2:])
        per = y.element_size() * (1 if not tail else _prod(tail))
        chunks, n = [], 0
        for c in self.tokens:
            chunks.append(y[n:n + c])
            n += c
        nr = self.n1 - self.n0
        got = _a2a_bytes(chunks, [nr * c * per for c in self.head_counts], self.group)
        return _cat([g.view(y.dtype).view(nr, c, *tail) for g, c in zip(got, self.head_counts)], 1)

    def head_major_to_heads(self, x):
        """[H][N_r][...] token shard (offsets, lse) -> [H_r][N][...] head shard."""
        if self.world == 1:
            return x
        tail = tuple(x.shape[2:])
        per = x.element_size() * (1 if not tail else _prod(tail))
        chunks, h = [], 0
        for c in self.head_counts:
            chunks.append(x[h:h + c])
            h += c
        hr = self.h1 - self.h0
        got = _a2a_bytes(chunks, [hr * n * per for n in self.tokens], self.group)
        return _cat([g.view(x.dtype).view(hr, n, *tail) for g, n in zip(got, self.tokens)], 1)

    def head_major_to_tokens(self, y):
        """[H_r][N][...] head shard -> [H][N_r][...] token shard."""
        if self.world == 1:
            return y
        tail = tuple(y.shape[2:])
        per = y.element_size() * (1 if not tail else _prod(tail))
        chunks, n = [], 0
        for c in self.tokens:
            chunks.append(y[:, n:n + c])
            n += c
        nr = self.n1 - self.n0
        got = _a2a_bytes(chunks, [c * nr * per for c in self.head_counts], self.group)
        return _cat([g.view(y.dtype).view(c, nr, *tail) for g, c in zip(got, self.head_counts)], 0)

    # --- the operator -------------------------------------------------------------------------
    def _check(self, q, offsets):
        nr, H = self.n1 - self.n0, self.heads
        if q.dim() != 3 or q.shape[0] != nr or q.shape[1] != H:
            raise ValueError(f"q must be this rank's token shard [{nr}][{H}][dh], got {tuple(q.shape)}")
        want = (H, nr, self.K, 3) if self.per_tap else (H, nr, 3)
        if tuple(offsets.shape) != want:
            raise ValueError(f"offsets must be {want}, got {tuple(offsets.shape)}")

    def forward(self, q, k, v, offsets):
        """Token shards in, token shards out: (out [N_r][H][dh], lse [H][N_r], ctx); ctx keeps the
        head-sharded inputs and lse for backward()."""
        self._check(q, offsets)
        qh, kh, vh = (self.rows_to_heads(t) for t in (q, k, v))
        oh = self.head_major_to_heads(offsets)
        out_h, lse_h = self.forward_fn(qh, kh, vh, oh, self.dims, self.window)
        ctx = (qh, kh, vh, oh, lse_h)
        return self.rows_to_tokens(out_h), self.head_major_to_tokens(lse_h), ctx

    def backward(self, ctx, dout):
        """dO token shard [N_r][H][dh] -> (dq, dk, dv [N_r][H][dh], doffsets [H][N_r][3] or
        [H][N_r][K][3])."""
        qh, kh, vh, oh, lse_h = ctx
        doh = self.rows_to_heads(dout)
        dq, dk, dv, doff = self.backward_fn(qh, kh, vh, oh, lse_h, doh, self.dims, self.window)
        return (self.rows_to_tokens(dq), self.rows_to_tokens(dk), self.rows_to_tokens(dv),
                self.head_major_to_tokens(doff))


def _prod(t):
    p = 1
    for x in t:
        p *= x
    return p


def _cat(parts, dim):
    import torch
    return torch.cat(parts, dim).contiguous()
