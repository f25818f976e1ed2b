"""Sink / local / update-buffer layout for long decoding.

ParisKV keeps recent tokens dense while older tokens are indexed and
offloaded (README, section on long generation: a sink/local/update-buffer
layout; slides, Fig. 5: sink and recent local tokens stay on the GPU for
dense attention, new tokens enter an update buffer, and a full buffer
triggers encoding and offload of the oldest local tokens; attention runs over
sink, local and retrieved tokens).  This module is that policy, written on
the library's C-ABI (pk_build_index, pk_append, pk_search, pk_attend_dense):
encoding, retrieval and attention run in the library's kernels; the buffer
bookkeeping (placing a new token in the dense buffer, moving the tail after
re-indexing) is plain tensor copies.

Positions 0 .. T-1 of every (sequence, KV head) pair are split into
  sink             [0, sink)             kept on the GPU, attended densely;
  retrieval zone   [sink, z)             in the ParisKV index (codes and
                                         records on the GPU, K/V in the index
                                         store -- pinned host memory when
                                         offloaded); searched for the Top-k;
  dense tail       [z, T)                kept on the GPU, attended densely.
The tail holds between `local` and `local + update` tokens.  When a new token
would make it longer, its oldest `update` tokens are encoded into the index
with one pk_append, and the zone grows by `update`.  Where the pages leave
the boundary rule open, this is the reading: re-indexing moves exactly
`update` tokens at a time and never lets the tail drop below `local`.

With async_reindex=True the batch is indexed off the decode stream (the
pages index and offload older tokens in the background): when the tail is
full, the oldest `update` tail tokens are staged with pk_append_stage on a
side stream, in `stage_pieces` pieces over as many consecutive steps, read
in place from the dense buffer, while the decode stream keeps attending them
densely.  The side stream also copies the tail rows that stay into a second
dense buffer, and new tokens go to both buffers meanwhile.  `publish_lag`
steps after the last piece, pk_append_publish makes the batch part of the
index on the decode stream (which waits for the side stream on the GPU, not
on the host) and the buffers swap.  The tail then holds up to
`local + update + stage_pieces - 1 + publish_lag` tokens.
"""
from __future__ import annotations

import torch

from . import (PK_BF16, PK_F32, PK_KV_DEVICE, PK_KV_HOST_PINNED, pk_append, pk_append_publish,
               pk_append_stage, pk_attend_dense, pk_build_index, pk_default_params, pk_free, pk_get_info,
               pk_search)


class ReindexPlan:
    """Which tokens move from the dense tail into the index, and when (pure
    bookkeeping: no tensors, no GPU).  before_token() is called at the start
    of a decode step, before the step's token joins the tail, and returns the
    step's actions, each with the tail length it saw:
      ("reindex", tail)             in line: pk_append of the oldest `update`
                                    tail tokens;
      ("stage", first, count, tail) stage tail tokens first .. first+count-1
                                    (counted from the tail's start); tail is
                                    given with the batch's first piece, when
                                    the surviving tail rows are copied, else
                                    None;
      ("publish",)                  the staged batch joins the index.
    add_token() then records the step's token."""

    def __init__(self, local: int, update: int, async_reindex: bool = False, pieces: int = 4,
                 publish_lag: int = 1):
        self.local, self.update = int(local), int(update)
        self.async_reindex = bool(async_reindex)
        # A batch is staged and published over pieces + lag steps while as many
        # tokens arrive; the tail only stays bounded if that is at most `update`.
        if self.async_reindex and self.update < 2:
            raise ValueError("asynchronous re-indexing needs update >= 2")
        self.lag = max(1, min(int(publish_lag), self.update - 1))
        self.pieces = max(1, min(int(pieces), self.update - self.lag))
        self.tail = self.local           # dense tail length
        self.published = 0               # tokens moved from the tail into the index
        self.reindexed = 0               # batches moved
        self.staged_for = -1             # steps since the batch's staging began, -1: none
        self.staged = 0                  # tokens of the batch staged so far

    @property
    def max_tail(self) -> int:
        extra = (self.pieces - 1 + self.lag) if self.async_reindex else 0
        return self.local + self.update + extra

    @property
    def staging(self) -> bool:
        return self.async_reindex and self.staged_for >= 0

    def before_token(self):
        acts = []
        u = self.update
        if self.async_reindex:
            if self.staged_for < 0 and self.tail >= self.local + u:
                self.staged_for = 0                       # a batch begins
            elif self.staged_for >= 0:
                self.staged_for += 1
            if self.staged_for >= 0 and self.staged_for >= self.pieces - 1 + self.lag:
                acts.append(("publish",))
                self.tail -= u
                self.published += u
                self.reindexed += 1
                self.staged_for = -1
                self.staged = 0
            elif self.staged_for >= 0 and self.staged_for < self.pieces:
                c = (u * (self.staged_for + 1)) // self.pieces - self.staged
                acts.append(("stage", self.staged, c, self.tail if self.staged == 0 else None))
                self.staged += c
        elif self.tail == self.local + u:
            acts.append(("reindex", self.tail))
            self.tail -= u
            self.published += u
            self.reindexed += 1
        return acts

    def add_token(self):
        self.tail += 1
        if self.tail > self.max_tail:
            raise RuntimeError("dense tail past its capacity")


class DecodeCache:
    """K, V: the prefill [batch][H][T0][D] (bf16 or fp32, on the GPU).
    sink, local, update: the layout sizes (pages: sink 4-64, local 256-512,
    update interval 256-512).  max_len: the largest T the cache will see
    (sizes the index).  The index is built over [sink, T0 - local), which
    must hold at least `topk` tokens."""

    def __init__(self, K, V, *, group: int, sink: int = 64, local: int = 512, update: int = 512,
                 max_len: int, topk: int = 100, offload: bool = False, async_reindex: bool = False,
                 publish_lag: int = 1, stage_pieces: int = 4, **params):
        assert K.dim() == 4 and K.shape == V.shape and K.shape[-1] == 128
        self.batch, self.H, T0, D = K.shape
        self.G, self.sink, self.local, self.update, self.topk = group, sink, local, update, topk
        if T0 - sink - local < max(1, topk):
            raise ValueError("the prefill must be longer than sink + local + topk tokens")
        self.dtype = K.dtype
        z = T0 - local                                    # zone end
        p = pk_default_params(batch=self.batch, n_kv_heads=self.H, group=group, topk=topk,
                              n_cap=max(max_len - sink - local, z - sink),
                              kv_dtype=PK_BF16 if K.dtype == torch.bfloat16 else PK_F32,
                              kv_location=PK_KV_HOST_PINNED if offload else PK_KV_DEVICE, **params)
        self.index = pk_build_index(K[:, :, sink:z].contiguous(), V[:, :, sink:z].contiguous(), z - sink, p)
        self.async_reindex = async_reindex
        self.plan = ReindexPlan(local, update, async_reindex, stage_pieces, publish_lag)
        cap = sink + self.plan.max_tail
        self.cap = cap
        self.dK = torch.zeros(self.batch, self.H, cap, D, dtype=K.dtype, device=K.device)
        self.dV = torch.zeros_like(self.dK)
        self.dK[:, :, :sink] = K[:, :, :sink]
        self.dV[:, :, :sink] = V[:, :, :sink]
        self.dK[:, :, sink:sink + local] = K[:, :, z:]
        self.dV[:, :, sink:sink + local] = V[:, :, z:]
        if async_reindex:
            # the second dense buffer (the sink rows never change) and the staging stream
            self.dK2 = self.dK.clone()
            self.dV2 = self.dV.clone()
            self.side = torch.cuda.Stream(device=K.device)
        self.T = T0
        self.zone_start_end = z                           # zone end at build
        self.idx = torch.empty(self.batch * self.H, topk, dtype=torch.int32, device=K.device)
        self.out = torch.empty(self.batch, self.H * group, D, dtype=torch.float32, device=K.device)

    @property
    def zone(self):
        """(start, end) positions of the retrieval zone."""
        return self.sink, self.zone_end

    @property
    def zone_end(self):
        return self.zone_start_end + self.plan.published

    @property
    def tail(self):
        """Dense tail length."""
        return self.plan.tail

    @property
    def reindexed(self):
        """Batches moved from the tail into the index."""
        return self.plan.reindexed

    @property
    def staged_for(self):
        return self.plan.staged_for

    def _reindex(self, tail):
        s, u = self.sink, self.update
        pk_append(self.index, self.dK[:, :, s:s + u].contiguous(), self.dV[:, :, s:s + u].contiguous(), u)
        rest = tail - u
        self.dK[:, :, s:s + rest] = self.dK[:, :, s + u:s + tail].clone()
        self.dV[:, :, s:s + rest] = self.dV[:, :, s + u:s + tail].clone()

    def _stage_piece(self, first, count, tail):
        """Stage tail tokens first .. first+count-1 on the side stream, in
        place; with the batch's first piece (tail given), copy the tail rows
        that stay into the second buffer."""
        s, u = self.sink, self.update
        self.side.wait_stream(torch.cuda.current_stream())   # rows written on the decode stream
        if tail is not None:
            with torch.cuda.stream(self.side):
                rest = tail - u
                self.dK2[:, :, s:s + rest].copy_(self.dK[:, :, s + u:s + tail])
                self.dV2[:, :, s:s + rest].copy_(self.dV[:, :, s + u:s + tail])
        r0 = s + first
        pk_append_stage(self.index, self.dK[:, :, r0:], self.dV[:, :, r0:], count, self.cap, stream=self.side)

    def _publish(self):
        """Make the staged tokens part of the index; the second buffer, which
        holds the surviving tail, takes over."""
        pk_append_publish(self.index)                     # the decode stream waits for the staging
        self.dK, self.dK2 = self.dK2, self.dK
        self.dV, self.dV2 = self.dV2, self.dV

    def step(self, q, k_new, v_new):
        """One decode step: add the new token k_new, v_new [batch][H][1][D] to
        the dense tail (re-indexing first when the buffer is full), retrieve
        the zone's Top-k for q [batch][H*G][D], and attend over sink + tail +
        retrieved rows.  Returns the attention output [batch][H*G][D] fp32
        (a buffer reused by the next step).  Everything runs on torch's current
        stream, in order, except the asynchronous staging."""
        for act in self.plan.before_token():
            if act[0] == "reindex":
                self._reindex(act[1])
            elif act[0] == "stage":
                self._stage_piece(act[1], act[2], act[3])
            else:
                self._publish()
        r = self.sink + self.plan.tail
        self.dK[:, :, r:r + 1] = k_new
        self.dV[:, :, r:r + 1] = v_new
        if self.plan.staging:                             # also into the buffer that takes over
            self.dK2[:, :, r - self.update:r - self.update + 1] = k_new
            self.dV2[:, :, r - self.update:r - self.update + 1] = v_new
        self.plan.add_token()
        self.T += 1
        pk_search(self.index, q, self.topk, self.idx)
        pk_attend_dense(self.index, q, self.idx, self.topk, self.dK, self.dV, self.sink + self.plan.tail, self.out)
        return self.out

    def close(self):
        if self.index is not None:
            if self.async_reindex:
                self.side.synchronize()               # no staging work in flight
            pk_free(self.index)
            self.index = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def info(self):
        return pk_get_info(self.index)
