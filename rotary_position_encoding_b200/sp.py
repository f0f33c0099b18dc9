"""Multi-GPU wiring of the sequence-parallel step (``rope3d_qk_norm_rope_append_sp``) and
of the exchange back after attention (``rope3d_sp_output_all_to_all``).

One process per GPU.  Every rank owns, in one symmetric-memory allocation that all ranks
of the group map, the buffers the step writes for its heads: q [B, q_rows, N/P, 128] and
the K and V caches [B, C, N/P, 128] (head-major: [B, N/P, C, 128]), and the buffer the
output exchange writes for its token slice, [B, rows, N, 128].  The table of every
rank's addresses (rank order) lets each rank's step store each head of its own token
slice straight into the owner's buffers over NVLink ("Accelerating Video Generation
Inference with Sequential-Parallel 3D Positional Encoding Using a Global Time Index",
Algorithm 3 steps 3-5 with the FusedAllToAll of Section 3.4.1 item 1 folded into the
stores), and lets the output exchange (Algorithm 3, last step) send each token of this
rank's heads back to the rank whose slice holds it.  After either, ``barrier()`` orders
every rank's reads of its own buffers after all ranks' stores.

Only argument marshalling and address bookkeeping happen here; the work is the CUDA
library's.  The allocation and the exchange of base addresses go through
``torch.distributed._symmetric_memory`` by default; ``exchange`` can be replaced (the
CPU tests pass one built on ``all_gather_object``).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import rope3d

HEAD_DIM = 128
_ALIGN = 256  # byte alignment of each region inside the allocation
BARRIER_TIMEOUT_MS = 10_000


def _align(n: int) -> int:
    return (n + _ALIGN - 1) // _ALIGN * _ALIGN


@dataclass
class Layout:
    """Byte offsets of a rank's four regions inside its allocation."""
    q_shape: tuple
    cache_shape: tuple
    elem: int
    q_off: int
    k_off: int
    v_off: int
    out_off: int          # output of the exchange after attention: [B, rows, N, 128]
    out_rows: int         # room for the largest token slice
    nbytes: int


def even_cuts(L: int, P: int):
    """Token slices [cuts[r], cuts[r+1]) of P ranks over L tokens: r L // P."""
    return [(r * L) // P for r in range(P + 1)]


def plan(B: int, N: int, P: int, q_rows: int, cache_tokens: int, dtype: torch.dtype,
         cache_layout: int = rope3d.ROPE3D_CACHE_TOKEN_MAJOR, out_rows: int | None = None
         ) -> Layout:
    """The allocation of one rank (the same on every rank).  out_rows defaults to the
    largest slice of the even split of q_rows tokens."""
    if N % P:
        raise ValueError(f"N={N} heads do not split evenly over {P} ranks")
    hl = N // P
    elem = torch.empty((), dtype=dtype).element_size()
    q_shape = (B, q_rows, hl, HEAD_DIM)
    cache_shape = ((B, cache_tokens, hl, HEAD_DIM) if cache_layout == rope3d.ROPE3D_CACHE_TOKEN_MAJOR
                   else (B, hl, cache_tokens, HEAD_DIM))
    if out_rows is None:
        cuts = even_cuts(q_rows, P)
        out_rows = max(cuts[r + 1] - cuts[r] for r in range(P))
    q_bytes = B * q_rows * hl * HEAD_DIM * elem
    c_bytes = B * cache_tokens * hl * HEAD_DIM * elem
    o_bytes = B * out_rows * N * HEAD_DIM * elem
    q_off = 0
    k_off = _align(q_off + q_bytes)
    v_off = _align(k_off + c_bytes)
    out_off = _align(v_off + c_bytes)
    return Layout(q_shape, cache_shape, elem, q_off, k_off, v_off, out_off, out_rows,
                  _align(out_off + o_bytes))


def symmetric_exchange(nbytes: int, device, group):
    """Allocate ``nbytes`` of symmetric memory on this rank and map every rank's
    allocation: returns (local uint8 tensor, [base address of rank r's allocation as seen
    from this process], barrier callable)."""
    import torch.distributed._symmetric_memory as symm_mem
    buf = symm_mem.empty(nbytes, dtype=torch.uint8, device=device)
    handle = symm_mem.rendezvous(buf, group)
    shift = buf.data_ptr() - handle.buffer_ptrs[handle.rank]  # the tensor's offset
    bases = [int(p) + shift for p in handle.buffer_ptrs]

    def barrier():
        handle.barrier(channel=0, timeout_ms=BARRIER_TIMEOUT_MS)  # bounded device wait

    return buf, bases, barrier


class SequenceParallelStep:
    """This rank's destination buffers and the step that writes every rank's."""

    def __init__(self, group, rank: int, world: int, B: int, N: int, q_rows: int,
                 cache_tokens: int, dtype: torch.dtype, device,
                 cache_layout: int = rope3d.ROPE3D_CACHE_TOKEN_MAJOR, q_row0: int = 0,
                 out_rows: int | None = None, exchange=symmetric_exchange):
        if not 1 <= world <= rope3d.ROPE3D_SP_MAX_RANKS:
            raise ValueError(f"1 to {rope3d.ROPE3D_SP_MAX_RANKS} ranks")
        self.rank, self.world, self.B, self.N = rank, world, B, N
        self.q_rows, self.cache_tokens, self.q_row0 = q_rows, cache_tokens, q_row0
        self.cache_layout, self.dtype = cache_layout, dtype
        self.layout = plan(B, N, world, q_rows, cache_tokens, dtype, cache_layout, out_rows)
        lay = self.layout
        self.buffer, bases, self._barrier = exchange(lay.nbytes, device, group)
        if len(bases) != world:
            raise RuntimeError("the exchange returned one address per rank")

        def view(off, shape):
            n = 1
            for d in shape:
                n *= d
            return self.buffer[off:off + n * lay.elem].view(dtype).view(shape)

        # this rank's own regions, as tensors
        self.q = view(lay.q_off, lay.q_shape)
        self.k_cache = view(lay.k_off, lay.cache_shape)
        self.v_cache = view(lay.v_off, lay.cache_shape)
        # every rank's regions, as addresses valid in this process
        self.q_dst = [b + lay.q_off for b in bases]
        self.k_dst = [b + lay.k_off for b in bases]
        self.v_dst = [b + lay.v_off for b in bases]
        self.out_dst = [b + lay.out_off for b in bases]
        self._view = view

    def out(self, rows: int):
        """This rank's output region as [B, rows, N, 128] (rows = its token slice)."""
        if not 0 <= rows <= self.layout.out_rows:
            raise ValueError(f"{rows} rows do not fit the {self.layout.out_rows}-row region")
        return self._view(self.layout.out_off, (self.B, rows, self.N, HEAD_DIM))

    def output_all_to_all(self, o, cuts=None, stream=None):
        """Algorithm 3's last step: o [B, L, N/P, 128] (attention's output for this rank's
        heads, every token) goes token by token to the output region of the rank whose
        slice holds the token.  cuts defaults to the even split; returns this rank's
        output view (valid after ``barrier()``)."""
        L = o.shape[1]
        cuts = even_cuts(L, self.world) if cuts is None else list(cuts)
        for r in range(self.world):
            if cuts[r + 1] - cuts[r] > self.layout.out_rows:
                raise ValueError(f"rank {r}'s slice does not fit its output region")
        rope3d.rope3d_sp_output_all_to_all(o, self.out_dst, self.rank, cuts, stream=stream)
        return self.out(cuts[self.rank + 1] - cuts[self.rank])

    def step(self, q, k, v, token_begin: int, token_end: int, frame_offset: int, T: int,
             H: int, W: int, q_norm_w, k_norm_w, eps: float, slot: int, tables,
             trig: int = rope3d.ROPE3D_TRIG_TABLE, stream=None) -> None:
        """This rank's slice [token_begin, token_end): q, k, v are [B, n, N, 128]."""
        rope3d.rope3d_qk_norm_rope_append_sp(
            q, k, v, token_begin, token_end, frame_offset, T, H, W, q_norm_w, k_norm_w, eps,
            self.q_dst, self.k_dst, self.v_dst, slot, tables, trig, self.cache_layout,
            q_row0=self.q_row0, q_rows=self.q_rows, cache_tokens=self.cache_tokens,
            stream=stream)

    def barrier(self) -> None:
        """Order every rank's later work after all ranks' stores so far."""
        self._barrier()
