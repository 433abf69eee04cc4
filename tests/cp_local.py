"""All shards of a context-parallel decode batch in one process (one GPU): the phases of
long_context_sparse_05_b200.cp run shard by shard, with the two collectives done by
copies and a sum between the phases (no kernel waits on another)."""

import torch


class LocalGroup:
    def __init__(self, shards):
        self.shards = shards

    def step(self, stream=None):
        for s in self.shards:
            s.phase_local(stream)
        cs = torch.stack([s.cand_s for s in self.shards])
        ci = torch.stack([s.cand_i for s in self.shards])
        for s in self.shards:
            s.gath_s.copy_(cs)
            s.gath_i.copy_(ci)
        for s in self.shards:
            s.phase_merge(stream)
        # one shard holds each selected row, the others zeros: the sum is exact
        total = torch.stack([s.rows for s in self.shards]).float().sum(0).to(self.shards[0].rows.dtype)
        for s in self.shards:
            s.rows.copy_(total)
        return [s.phase_attend(stream) for s in self.shards]
