"""Continuous-batching trace driver over a paged block allocator.

The pages name continuous batching as the serving loop that paged memory
feeds ("pagedattention" glossary entry, paragraph 5) and beam search as a case
of sharing (its samples point at the same physical blocks and are copied on
write only when they diverge).  This module plays such a loop against an
allocator so the decode path can be measured and checked under it; it makes
no allocation decisions itself (those are the allocator's), it only decides
which sequences exist:

* requests arrive per the trace draws (synth.trace) and wait in FIFO order;
* a request is admitted when the free blocks cover its prompt plus a reserve;
  admission creates a root sequence, appends the prompt tokens, and forks
  beam - 1 more beams that share every prompt block;
* every step each running beam appends one token (the decode token);
* per step and running group, a Bernoulli draw replaces one beam (freed) by
  a fork of another beam of the group (beam re-selection);
* a group finishes after its drawn output length and frees its beams.

The same driver runs on the library's Allocator and on the oracle's model;
with the same draws both see the same operations in the same order.
"""
from __future__ import annotations

from collections import deque
from dataclasses import dataclass, field

import numpy as np


@dataclass
class StepPlan:
    """What one step asks of the device path, in order."""

    prompt_seqs: list          # sequences whose prompt rows are written this step
    prompt_slots: np.ndarray   # int64 slots of those prompt tokens, in order
    decode_seqs: list          # every running beam, decoded this step
    decode_slots: np.ndarray   # int64 slot of each beam's new token
    cow_pairs: np.ndarray      # int32 [k, 2] copy-on-write pairs of the decode appends
    forks: int = 0
    frees: int = 0


@dataclass
class _Group:
    beams: list
    left: int


@dataclass
class BeamTrace:
    alloc: object                 # new_seq / fork / free_seq / batch_append
    free_blocks: object           # callable -> number of free blocks
    block_size: int
    draws: list                   # synth.trace(...) output
    beam: int = 4
    reserve_blocks: int = 4
    max_running_beams: int = 1 << 30
    waiting: deque = field(default_factory=deque)
    running: list = field(default_factory=list)
    step_no: int = 0

    def _blocks_for(self, n_tokens: int) -> int:
        return -(-int(n_tokens) // self.block_size)

    def step(self) -> StepPlan:
        d = self.draws[self.step_no]
        self.step_no += 1
        frees = forks = 0
        # groups whose output is complete leave and free their beams
        keep = []
        for g in self.running:
            if g.left <= 0:
                for s in g.beams:
                    self.alloc.free_seq(s)
                    frees += 1
            else:
                keep.append(g)
        self.running = keep
        # beam re-selection: one beam of a group replaced by a fork of another
        for i, g in enumerate(self.running):
            if i < len(d["reselect"]) and d["reselect"][i]:
                v = int(d["victim"][i]) % self.beam
                donor = g.beams[(v + 1 + int(d["donor"][i])) % self.beam]
                self.alloc.free_seq(g.beams[v])
                g.beams[v] = self.alloc.fork(donor)
                frees += 1
                forks += 1
        # arrivals, then FIFO admission while the pool covers prompt + reserve
        self.waiting.extend(d["arrivals"])
        prompt_seqs, prompt_lens = [], []
        running_beams = self.beam * len(self.running)
        while self.waiting:
            plen, olen = self.waiting[0]
            need = self._blocks_for(plen) + self.reserve_blocks + running_beams + self.beam
            if self.free_blocks() < need or running_beams + self.beam > self.max_running_beams:
                break
            self.waiting.popleft()
            root = self.alloc.new_seq()
            slots, _ = self.alloc.batch_append([root], [plen])
            prompt_seqs.append(root)
            prompt_lens.append(np.asarray(slots, dtype=np.int64))
            beams = [root] + [self.alloc.fork(root) for _ in range(self.beam - 1)]
            forks += self.beam - 1
            self.running.append(_Group(beams=beams, left=int(olen)))
            running_beams += self.beam
        # the decode token of every running beam
        decode_seqs = [s for g in self.running for s in g.beams]
        if decode_seqs:
            slots, pairs = self.alloc.batch_append(decode_seqs, [1] * len(decode_seqs))
            slots = np.asarray(slots, dtype=np.int64)
            pairs = np.asarray(pairs, dtype=np.int32).reshape(-1, 2)
        else:
            slots, pairs = np.zeros(0, np.int64), np.zeros((0, 2), np.int32)
        for g in self.running:
            g.left -= 1
        return StepPlan(prompt_seqs=prompt_seqs,
                        prompt_slots=np.concatenate(prompt_lens) if prompt_lens else np.zeros(0, np.int64),
                        decode_seqs=decode_seqs, decode_slots=slots, cow_pairs=pairs, forks=forks, frees=frees)
