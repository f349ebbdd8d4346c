"""The layer over several GPUs: one process per GPU, ``torch.distributed`` for the plumbing.

Two partitions follow from the layer's structure ("Swimba: Switch Mamba Model Scales State Space
Models": one state trajectory per sequence; "Mamba y las SSMs: el retorno del estado persistente",
"Estado interno puramente lineal": the state is linear, so the recurrence can be cut and
recombined):

* **batch** -- sequences are independent. Rank r owns the contiguous block of sequences
  ``batch_shard(B, world, r)`` of the global batch; nothing crosses ranks on the data path.
* **sequence** -- one long sequence is cut into ``world`` consecutive pieces
  (``sequence_piece``). Every rank routes and projects its own tokens (token-local), summarises its
  piece (the end state from zero and the summed log decay, ``swimba_scan_summary``), one
  ``all_gather`` exchanges the [2, B, D, N] summaries (256 KB for D = 2048, N = 16), every rank
  chains them into its piece's start state (``swimba_scan_chain``), and scans its piece from there
  (``swimba_scan_fwd`` with that h0). The chain is the same fp32 arithmetic on every rank, so all
  ranks hold the same start states; the last entry is the state after the whole sequence.

The functions here hold no arithmetic of the layer: the summaries, the chain and the scan are
callables of an ``ops`` object (``CudaPieceOps`` runs the library's kernels through the C ABI).
"""
from __future__ import annotations

import ctypes


def batch_shard(batch: int, world: int, rank: int) -> tuple[int, int]:
    """[start, stop) of the sequences rank ``rank`` owns: contiguous, sizes differing by at most 1."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    return batch * rank // world, batch * (rank + 1) // world


def sequence_piece(seqlen: int, world: int, rank: int, align: int = 16) -> tuple[int, int]:
    """[start, stop) of the tokens rank ``rank`` owns when one sequence is cut into ``world``
    consecutive pieces. Cuts fall on multiples of ``align`` tokens (the scan's chunk), so every
    piece but the last is a whole number of chunks; pieces may be empty only when the sequence has
    fewer chunks than ranks."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    chunks = -(-seqlen // align)

    def cut(r):
        return min(seqlen, (chunks * r // world) * align)

    return cut(rank), cut(rank + 1)


def exchange_summaries(h_zero, log_decay, dist, group=None):
    """All-gather of every rank's piece summary: returns (h_zero_all, log_decay_all), each
    [world, *h_zero.shape], piece 0 (rank 0) first. The one collective of the sequence split."""
    import torch

    world = dist.get_world_size(group)
    packed = torch.stack([h_zero, log_decay]).contiguous()
    out = torch.empty((world,) + tuple(packed.shape), dtype=packed.dtype, device=packed.device)
    dist.all_gather(list(out.unbind(0)), packed, group=group)
    return out[:, 0], out[:, 1]


def sequence_parallel_scan(ops, piece, dist, h0=None, group=None):
    """The sequence split on this rank: summary of the local piece, one exchange, the chain into
    start states, the scan of the local piece from its start state.

    ``ops.summary(piece) -> (h_zero, log_decay)``; ``ops.chain(h_zero_all, log_decay_all, h0) ->
    h_start [world + 1, ...]``; ``ops.scan(piece, h_start_of_this_piece) -> result``.
    Returns (result, h_after_the_whole_sequence)."""
    rank = dist.get_rank(group)
    h_zero, log_decay = ops.summary(piece)
    hz_all, ld_all = exchange_summaries(h_zero, log_decay, dist, group)
    h_start = ops.chain(hz_all, ld_all, h0)
    return ops.scan(piece, h_start[rank]), h_start[-1]


class CudaPieceOps:
    """The sequence split's three steps on the library's kernels (device tensors, one stream).

    A piece is a ``LayerBuffers`` already filled by route and mixed projection for the rank's
    tokens, plus its x and z: ``piece = (dims, x, z, buf)``."""

    def __init__(self, S, weights_struct, stream=None):
        self.S, self.w, self.stream = S, weights_struct, stream

    def summary(self, piece):
        import torch

        S = self.S
        dims, x, _, buf = piece
        B, D, N = dims.batch, dims.d_inner, dims.d_state
        h_zero = torch.empty((B, D, N), dtype=torch.float32, device=x.device)
        log_decay = torch.empty_like(h_zero)
        ws = S.new_workspace(dims, S.SWIMBA_OP_SUMMARY, x.device)
        S.check(S.swimba_scan_summary(dims, x, buf.delta, buf.B_mix, buf.idx, buf.gates, self.w, h_zero, log_decay,
                                      ws, ws.numel(), self.stream), "swimba_scan_summary")
        return h_zero, log_decay

    def chain(self, h_zero_all, log_decay_all, h0):
        import torch

        P = h_zero_all.shape[0]
        h_start = torch.empty((P + 1,) + tuple(h_zero_all.shape[1:]), dtype=torch.float32, device=h_zero_all.device)
        dims = self.S.swimba_dims(batch=h_zero_all.shape[1], seqlen=1, d_inner=h_zero_all.shape[2],
                                  d_state=h_zero_all.shape[3], dt_rank=1, n_experts=1, top_k=1)
        self.S.check(self.S.swimba_scan_chain(dims, P, h_zero_all.contiguous(), log_decay_all.contiguous(), h0,
                                              h_start, self.stream), "swimba_scan_chain")
        return h_start

    def scan(self, piece, h_start):
        S = self.S
        dims, x, z, buf = piece
        S.check(S.swimba_scan_fwd(dims, x, z, buf.delta, buf.B_mix, buf.C_mix, buf.idx, buf.gates, self.w,
                                  h_start.contiguous(), buf.out, buf.h_final, buf.y, buf.ws, buf.ws.numel(),
                                  self.stream), "swimba_scan_fwd")
        return buf

    def route_and_project(self, piece):
        S = self.S
        dims, x, _, buf = piece
        S.check(S.swimba_route(dims, x, ctypes.c_void_p(self.w.W_r).value, buf.idx, buf.gates, self.stream),
                "swimba_route")
        S.check(S.swimba_mixed_proj(dims, x, buf.idx, buf.gates, self.w, buf.delta, buf.B_mix, buf.C_mix, buf.ws,
                                    buf.ws.numel(), self.stream), "swimba_mixed_proj")
