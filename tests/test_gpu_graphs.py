"""The decode step captured in a CUDA graph and replayed, as a serving loop
would run it. The per-segment piece counters are tagged with an epoch that the
kernels advance in the workspace header at the end of every launch, so each
replay -- whose launch parameters are frozen at capture -- still has an epoch
of its own. Replays are checked bit for bit against eager calls and against
the fp64 oracle, on batches whose contexts are cut into merged pieces.
"""
import pytest
import torch

import oracle
import paged_kv_cache_377_b200 as pkv
import workloads
from helpers import assert_close_to_oracle

pytestmark = pytest.mark.gpu

DEV = "cuda"


class Step:
    """Static device buffers of one fused decode step (append + attention)."""

    def __init__(self, b, **opts):
        self.b = b
        self.kc = b.k_cache.to(DEV, copy=True)
        self.vc = b.v_cache.to(DEV, copy=True)
        self.q = b.q.to(DEV, copy=True)
        self.kn = b.k_new.to(DEV)
        self.vn = b.v_new.to(DEV)
        self.slots = b.slot_mapping.to(DEV)
        self.bt = b.block_tables.to(DEV)
        self.cl = b.context_lens.to(DEV)
        self.ws = pkv.allocate_workspace(b.num_seqs, b.num_q_heads, b.head_dim)
        self.out = torch.full_like(self.q, float("nan"))
        self.opts = opts

    def __call__(self):
        pkv.paged_attn_decode_append(self.out, self.q, self.kn, self.vn, self.slots, self.kc, self.vc, self.bt,
                                     self.cl, self.b.scale, self.ws, **self.opts)


def eager(b, q=None, **opts):
    st = Step(b, **opts)
    if q is not None:
        st.q.copy_(q)
    st()
    torch.cuda.synchronize()
    assert pkv.read_status(st.ws) == 0
    return st.out.cpu()


def capture(st):
    st()  # warm up outside the capture (first-call setup of the kernel)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        st()
    return g


@pytest.mark.parametrize("name,opts", [("skewed_long", {}), ("skewed_long", dict(num_ctas=1024)),
                                       ("llama3_8b", {}), ("opt125m", dict(num_ctas=700))])
def test_replays_of_a_captured_step_match_eager_calls_bitwise(name, opts):
    device = "cuda" if name in ("llama3_8b", "skewed_long") else "cpu"
    b = workloads.make_batch(name, device=device).to("cpu")
    want = eager(b, **opts)
    st = Step(b, **opts)
    g = capture(st)
    for _ in range(3):
        st.out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(st.out.cpu().view(torch.int16), want.view(torch.int16)), "a replay differs"
    assert pkv.read_status(st.ws) == 0


def test_replays_with_new_queries_match_the_oracle():
    """New q between replays (the static buffer is refilled), as the next
    decode step of a served batch would be."""
    b = workloads.make_batch("skewed_long", device="cuda").to("cpu")
    st = Step(b)
    g = capture(st)
    gen = torch.Generator().manual_seed(7)
    for _ in range(2):
        q = torch.randn(b.q.shape, generator=gen).to(torch.bfloat16)
        st.q.copy_(q)
        g.replay()
        torch.cuda.synchronize()
        nb = workloads.DecodeBatch(**{**b.__dict__, "q": q})
        pairs = list(range(0, nb.num_seqs * nb.num_q_heads, 11))
        ref, _, _ = oracle.decode_step(nb, pairs=pairs)
        got = st.out.cpu().double().numpy().reshape(-1, nb.head_dim)[pairs]
        assert_close_to_oracle(got, ref, what="skewed_long replay with new q")
        assert torch.equal(st.out.cpu().view(torch.int16), eager(b, q=q).view(torch.int16))


def test_replays_with_prefix_groups_match_eager_calls_bitwise():
    """The launch with prefix groups is cooperative; it replays like any other."""
    b = workloads.make_batch("qwen25_7b_prefix")
    groups = pkv.find_prefix_groups(b.block_tables, b.context_lens, b.block_size)
    assert len(groups) == 1
    want = eager(b, prefix_groups=groups)
    st = Step(b, prefix_groups=groups)
    g = capture(st)
    for _ in range(3):
        st.out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(st.out.cpu().view(torch.int16), want.view(torch.int16)), "a replay differs"
    assert pkv.read_status(st.ws) == 0


def test_a_workspace_reused_by_many_calls_keeps_every_result():
    """Ten calls on one workspace, alternating batch shapes (their segments
    overlap in the counter array): each call's result equals a fresh one's."""
    a = workloads.make_batch("skewed_long", device="cuda").to("cpu")
    c = workloads.make_batch("opt125m")
    want_a, want_c = eager(a), eager(c)
    ws = pkv.allocate_workspace(max(a.num_seqs, c.num_seqs), max(a.num_q_heads, c.num_q_heads),
                                max(a.head_dim, c.head_dim))
    for i in range(10):
        b, want = (a, want_a) if i % 2 == 0 else (c, want_c)
        st = Step(b)
        st.ws = ws
        st()
        torch.cuda.synchronize()
        assert torch.equal(st.out.cpu().view(torch.int16), want.view(torch.int16)), f"call {i}"
    assert pkv.read_status(ws) == 0


def test_a_prepared_call_matches_the_plain_call_bitwise():
    """DecodeAppendCall launches the same step as paged_attn_decode_append; with
    its buffers refilled between calls it gives each new step's result."""
    b = workloads.make_batch("skewed_long", device="cuda").to("cpu")
    st = Step(b)
    call = pkv.DecodeAppendCall(st.out, st.q, st.kn, st.vn, st.slots, st.kc, st.vc, st.bt, st.cl, b.scale, st.ws)
    gen = torch.Generator().manual_seed(3)
    for _ in range(2):
        q = torch.randn(b.q.shape, generator=gen).to(torch.bfloat16)
        st.q.copy_(q)
        st.out.fill_(float("nan"))
        call()
        torch.cuda.synchronize()
        assert torch.equal(st.out.cpu().view(torch.int16), eager(b, q=q).view(torch.int16))
    assert pkv.read_status(st.ws) == 0

