"""A synthetic continuous-batching stream driven through the block manager.

Sequences join (prompt tokens, some starting with another sequence's prompt
blocks), fork (parallel sampling / beam search), take decode steps and leave,
as runbyai post 449 (sections 3-4) and "Deep Dive into vLLM" (section 2.2)
describe. Ground truth is kept the plain way: each sequence's K/V rows in
logical order, as Python lists. A backend applies the pool writes the stream
asks for (prompt tokens at their slots, copy-on-write block copies) so the
paged pool can be checked against the truth.
"""
from __future__ import annotations

import numpy as np
import torch


class HostPool:
    """The pool as bf16 CPU tensors; writes and copies done with plain indexing."""

    def __init__(self, num_blocks, block_size, num_kv_heads, head_dim):
        shape = (num_blocks, block_size, num_kv_heads, head_dim)
        self.k = torch.full(shape, float("nan"), dtype=torch.bfloat16)
        self.v = torch.full(shape, float("nan"), dtype=torch.bfloat16)
        self.bs = block_size

    def write(self, slots, k_rows, v_rows):
        for i, s in enumerate(slots):
            if s >= 0:
                self.k[s // self.bs, s % self.bs] = k_rows[i]
                self.v[s // self.bs, s % self.bs] = v_rows[i]

    def copy_blocks(self, src, dst):
        for a, b in zip(src, dst):
            self.k[b] = self.k[a]
            self.v[b] = self.v[a]


class Stream:
    def __init__(self, bm, num_kv_heads, head_dim, num_q_heads, seed):
        self.bm = bm
        self.Hkv, self.D, self.Hq = num_kv_heads, head_dim, num_q_heads
        self.rng = np.random.default_rng(seed)
        self.gen = torch.Generator().manual_seed(seed)
        self.truth = {}      # seq id -> ([K rows], [V rows]) in logical order, each bf16 [Hkv][D]
        self.next_id = 0

    def _rows(self, n):
        k = torch.randn(n, self.Hkv, self.D, generator=self.gen).to(torch.bfloat16)
        v = torch.randn(n, self.Hkv, self.D, generator=self.gen).to(torch.bfloat16)
        return k, v

    def join(self, n, prefix_of=None, prefix_tokens=0):
        """A new sequence with an n-token prompt; returns (id, slots, k, v) of the prompt's
        tokens to write (slots -1 for tokens in shared blocks)."""
        sid = self.next_id
        self.next_id += 1
        slots = self.bm.add(sid, n, -1 if prefix_of is None else prefix_of,
                            prefix_tokens if prefix_of is not None else 0)
        k, v = self._rows(n)
        if prefix_of is not None:  # the prompt starts with the other sequence's tokens
            pk, pv = self.truth[prefix_of]
            shared = (prefix_tokens // self.bm.block_size) * self.bm.block_size
            for t in range(prefix_tokens):
                k[t], v[t] = pk[t], pv[t]
            assert np.all(slots[:shared] == -1) and np.all(slots[shared:] >= 0)
        self.truth[sid] = ([k[t] for t in range(n)], [v[t] for t in range(n)])
        return sid, slots, k, v

    def fork(self, parent):
        sid = self.next_id
        self.next_id += 1
        self.bm.fork(parent, sid)
        pk, pv = self.truth[parent]
        self.truth[sid] = (list(pk), list(pv))
        return sid

    def leave(self, sid):
        self.bm.free(sid)
        del self.truth[sid]

    def step(self, ids, max_blocks):
        """One decode step of sequences `ids`: reserve each one's next slot (copy-on-
        write as needed), take the copies, pack the tables. Returns the step's inputs."""
        slots = np.array([self.bm.append(s) for s in ids], dtype=np.int64)
        src, dst = self.bm.take_copies()
        bt, cl = self.bm.pack(ids, max_blocks)
        k_new, v_new = self._rows(len(ids))
        q = torch.randn(len(ids), self.Hq, self.D, generator=self.gen).to(torch.bfloat16)
        for i, s in enumerate(ids):
            self.truth[s][0].append(k_new[i])
            self.truth[s][1].append(v_new[i])
        return dict(slots=slots, src=src, dst=dst, bt=bt, cl=cl, k_new=k_new, v_new=v_new, q=q)

    def reference(self, ids, q, scale):
        """Brute-force attention over each sequence's own token list (fp64)."""
        G = self.Hq // self.Hkv
        out = np.zeros((len(ids), self.Hq, self.D))
        for i, s in enumerate(ids):
            K = torch.stack(self.truth[s][0]).double().numpy()  # [L][Hkv][D]
            V = torch.stack(self.truth[s][1]).double().numpy()
            for j in range(self.Hq):
                x = scale * K[:, j // G, :] @ q[i, j].double().numpy()
                w = np.exp(x - x.max())
                out[i, j] = (w[:, None] * V[:, j // G, :]).sum(0) / w.sum()
        return out


def random_stream(stream, pool_apply, step_apply, steps, max_blocks, max_running=12, seed=0):
    """Drives joins, forks, leaves and decode steps; `pool_apply(slots, k, v)` writes prompt
    tokens, `step_apply(ids, inputs)` runs one decode step and checks it. Returns the
    number of copy-on-write copies made."""
    rng = np.random.default_rng(seed)
    bs = stream.bm.block_size
    running = []
    copies = 0
    for it in range(steps):
        # joins: some with a prefix of a running sequence's prompt
        while len(running) < max_running and rng.random() < 0.6:
            n = int(rng.integers(1, 5 * bs))
            if running and rng.random() < 0.4:
                src = int(rng.choice(running))
                L = len(stream.truth[src][0])
                p = int(rng.integers(0, min(L, n) + 1))
                try:
                    sid, slots, k, v = stream.join(n, prefix_of=src, prefix_tokens=p)
                except Exception:
                    break
            else:
                try:
                    sid, slots, k, v = stream.join(n)
                except Exception:
                    break
            pool_apply(slots, k, v)
            running.append(sid)
        # forks (between steps)
        if running and rng.random() < 0.3 and len(running) < max_running + 4:
            running.append(stream.fork(int(rng.choice(running))))
        # leaves
        for s in list(running):
            if rng.random() < 0.08 or len(stream.truth[s][0]) + 1 >= max_blocks * bs:
                stream.leave(s)
                running.remove(s)
        if not running:
            continue
        # a decode step, if the pool can hold it
        if stream.bm.num_free < len(running) + 1:
            victim = running.pop(0)
            stream.leave(victim)
            if not running:
                continue
        inputs = stream.step(running, max_blocks)
        copies += len(inputs["src"])
        step_apply(list(running), inputs)
    return copies
