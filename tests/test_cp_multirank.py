"""Context-parallel selection across two and three gloo ranks on CPU, as torchrun would
start them.  Each rank holds one token-range shard of every sequence, and
hisa_cp_select's exchange (two all-gathers of (id, score) lists in rank order,
each merged by the rule score desc, id asc) must hand every rank the selection
of the whole sequence.  The library's per-shard steps need a GPU, so here
they are stood in for by a plain numpy restatement of the shard rules that
include/hisa.h states for hisa_cp_blocks, hisa_cp_tokens and hisa_merge_topk;
what is under test is the exchange.  The expected result is the oracle's
two-stage selection on the unsharded case."""
import json
import os
import socket
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
B, M, K = 64, 4, 64


def _shard_len(world):
    """Shards on block boundaries that together cover the 1024-token sequence."""
    return -(-1024 // (world * B)) * B


def _case():
    from hisa_inputs import make_case
    pos = [np.array([3, 100, 511, 512, 600, 1023]), np.array([40, 511, 699])]
    return make_case(batch=2, L=[1024, 700], H=4, d=64, B=B, m=M, k=K, positions=pos, seed=77)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class ShardSteps:
    """numpy stand-ins for the three library calls on the shard at tok_off."""

    def __init__(self, case, tok_off, lr):
        from hisa_inputs import bf16_to_f32
        self.keys = bf16_to_f32(case.keys).astype(np.float64)      # [batch, cap, d]
        self.tok_off = tok_off
        self.lr = lr
        self.n = np.clip(case.lens.astype(np.int64), tok_off, tok_off + lr) - tok_off

    def _score(self, Q, w, x):
        return float((np.maximum(Q @ x, 0.0) * w).sum())

    def _view(self, b, t):
        """(visible blocks, own) of the row on this shard, or None if invalid."""
        tl, n = t - self.tok_off, int(self.n[b])
        if tl < 0:
            return 0, 0
        if tl < n:
            return tl // B + 1, 1
        return (self.lr // B, 0) if n == self.lr else None

    def blocks(self, kv, tok_off, Q, w, qs, qp, m, ws=None):
        import torch
        Q, w = Q.double().numpy(), w.double().numpy()
        ids = np.full((len(qs), m), -1, np.int32)
        sc = np.full((len(qs), m), np.nan)
        for i, (b, t) in enumerate(zip(qs.tolist(), qp.tolist())):
            v = self._view(b, t)
            if v is None or v[0] == 0:
                continue
            vis, own = v
            s0, n = self.tok_off, int(self.n[b])
            score = {}
            for j in range(vis - own):
                mu = self.keys[b, s0 + j * B:s0 + min((j + 1) * B, n)].mean(axis=0)
                score[j] = self._score(Q[i], w[i], mu)
            keep = sorted(sorted(score, key=lambda j: (-score[j], j))[:m - 1])
            row = [(self.tok_off // B + j, score[j]) for j in keep]
            if own:
                row.append((self.tok_off // B + vis - 1, np.inf))
            for c, (g, s) in enumerate(row):
                ids[i, c], sc[i, c] = g, s
        return torch.from_numpy(ids), torch.from_numpy(sc)

    def tokens(self, kv, tok_off, Q, w, qs, qp, m, k, kept, ws=None):
        import torch
        Q, w, kept = Q.double().numpy(), w.double().numpy(), kept.numpy()
        idx = np.full((len(qs), k), -1, np.int32)
        sc = np.full((len(qs), k), np.nan)
        for i, (b, t) in enumerate(zip(qs.tolist(), qp.tolist())):
            v = self._view(b, t)
            if v is None or t // B not in kept[i] or v[0] == 0:
                continue
            vis, blk0 = v[0], self.tok_off // B
            cand = []
            for g in kept[i]:
                if blk0 <= g < blk0 + vis:
                    for s in range(g * B, min((g + 1) * B, t + 1)):
                        cand.append((-self._score(Q[i], w[i], self.keys[b, s]), s))
            top = sorted(sorted(cand)[:k], key=lambda e: e[1])
            for c, (s_neg, s) in enumerate(top):
                idx[i, c], sc[i, c] = s, -s_neg
        return torch.from_numpy(idx), torch.from_numpy(sc)

    @staticmethod
    def merge(ids, scores, k, stream=None):
        """As the kernel: slots in list-then-entry order, ties to the lower
        slot, output in slot order (so the lists must come in rank order)."""
        import torch
        ids, scores = ids.numpy(), scores.numpy()
        lists, rows, n = ids.shape
        out = np.full((rows, k), -1, np.int32)
        osc = np.full((rows, k), np.nan)
        for r in range(rows):
            ent = [(-float(scores[l, r, j]), l * n + j, int(ids[l, r, j]))
                   for l in range(lists) for j in range(n) if ids[l, r, j] >= 0]
            top = sorted(sorted(ent)[:k], key=lambda e: e[1])
            for c, (s, _, g) in enumerate(top):
                out[r, c], osc[r, c] = g, -s
        return torch.from_numpy(out), torch.from_numpy(osc)


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    import hierarchical_top_indexer_b200 as hisa
    dist.init_process_group("gloo", rank=rank, world_size=world)
    case = _case()
    lr = _shard_len(world)
    steps = ShardSteps(case, rank * lr, lr)
    hisa.hisa_cp_blocks, hisa.hisa_cp_tokens, hisa.hisa_merge_topk = steps.blocks, steps.tokens, steps.merge
    from hisa_inputs import bf16_to_f32
    Q = torch.from_numpy(bf16_to_f32(case.Q))
    idx, sc = hisa.hisa_cp_select(None, rank * lr, Q, torch.from_numpy(case.w),
                                  torch.from_numpy(case.q_seq), torch.from_numpy(case.q_pos), M, K)
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"idx": idx.tolist()}, f)


import pytest


@pytest.mark.parametrize("world", [2, 3])
def test_rank_exchange_gives_the_whole_sequence_selection(tmp_path, world):
    sys.path.insert(0, ROOT)
    from tests.test_abi import build_module
    build = build_module()
    if build.stale():
        build.build()
    import oracle
    case = _case()
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    got = [np.array(json.load(open(tmp_path / f"rank{r}.json"))["idx"]) for r in range(world)]
    ora = oracle.hisa_select(oracle.Cache.of(case), case.Q, case.w, case.q_seq, case.q_pos, B, M, K)
    for g in got:
        np.testing.assert_array_equal(g, ora["idx"])
