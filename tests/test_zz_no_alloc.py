"""paged_attn_decode_noalloc: decode without a caller-allocated workspace.

Some callers cannot allocate device memory at all: an engine that handed every
byte left after the weights to one preallocated KV pool, or a plugin host that
gives its plugins no allocator. They call paged_attn_decode_noalloc, whose
scratch is a static device array inside the library. These tests call it
through the C ABI and check it against paged_attn_decode, the entry point that
takes a workspace, on two calls in a row -- the second call must not be
disturbed by what the first left in the shared scratch.
"""
import pytest
import torch

import paged_kv_cache_377_b200 as pkv
import workloads
from helpers import assert_close_to_oracle

SCRATCH_BYTES = 64 << 20


def _decode_both(b, dev):
    kc, vc = b.k_cache.to(dev), b.v_cache.to(dev)
    q = b.q.to(dev)
    bt, cl = b.block_tables.to(dev), b.context_lens.to(dev)
    pkv.kv_cache_append(b.k_new.to(dev), b.v_new.to(dev), kc, vc, b.slot_mapping.to(dev))
    ws = pkv.allocate_workspace(b.num_seqs, b.num_q_heads, b.head_dim, device=dev)
    assert ws.numel() <= SCRATCH_BYTES
    with_ws = torch.empty_like(q)
    pkv.paged_attn_decode(with_ws, q, kc, vc, bt, cl, b.scale, ws)
    no_ws = torch.full_like(q, float("nan"))
    status = torch.full((1,), -1, dtype=torch.int32, device=dev)
    lib = pkv.library()
    from paged_kv_cache_377_b200._binding import paged_attn_decode_noalloc
    paged_attn_decode_noalloc(no_ws, q, kc, vc, bt, cl, b.scale, status=status)
    torch.cuda.synchronize()
    assert lib.pkv_last_error() == b""
    return with_ws.cpu(), no_ws.cpu(), int(status.item()), pkv.read_status(ws)


@pytest.mark.gpu
def test_noalloc_matches_the_workspace_entry_point_on_two_calls_in_a_row():
    dev = torch.device("cuda", torch.cuda.current_device())
    # the first call leaves split partials behind in the scratch; the second
    # has a different shape and cuts its contexts differently
    for name in ("llama3_8b", "opt125m"):
        b = workloads.make_batch(name, device=dev)
        with_ws, no_ws, status, ws_status = _decode_both(b, dev)
        assert status == 0 and ws_status == 0, (name, status, ws_status)
        # same kernel, options and grid: bit for bit (a stale partial left in the
        # scratch by the previous call could otherwise hide inside a tolerance)
        assert torch.equal(no_ws.view(torch.int16), with_ws.view(torch.int16)), f"noalloc vs workspace, {name}"
        assert_close_to_oracle(no_ws.double().numpy(), with_ws.double().numpy(), what=f"noalloc vs workspace, {name}")


@pytest.mark.gpu
def test_noalloc_status_reports_only_its_own_call():
    """d_status is overwritten per call: a call that meets a bad block id reports
    it, and the clean call after it, on the same scratch, reports 0."""
    dev = torch.device("cuda", torch.cuda.current_device())
    b = workloads.make_custom(81, [40, 40], 4, 2, 64, 16, with_append=False, poison=False, device=dev)
    q, kc, vc, cl = b.q, b.k_cache, b.v_cache, b.context_lens.to(dev)
    good = b.block_tables.to(dev)
    bad = good.clone()
    bad[1, 1] = b.num_blocks + 5
    from paged_kv_cache_377_b200._binding import paged_attn_decode_noalloc
    status = torch.full((1,), -1, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    paged_attn_decode_noalloc(out, q, kc, vc, bad, cl, b.scale, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == pkv.PKV_STATUS_BAD_BLOCK_ID
    paged_attn_decode_noalloc(out, q, kc, vc, good, cl, b.scale, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ws = pkv.allocate_workspace(b.num_seqs, b.num_q_heads, b.head_dim, device=dev)
    ref = torch.empty_like(q)
    pkv.paged_attn_decode(ref, q, kc, vc, good, cl, b.scale, ws)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_noalloc_rejects_batches_beyond_its_scratch():
    """2048 sequences of 64 query heads need ~100 MB of workspace: refused on the host, nothing enqueued."""
    lib = pkv.library()
    import ctypes
    P = ctypes.c_void_p(4096)
    from paged_kv_cache_377_b200._binding import paged_attn_decode_noalloc  # noqa: F401  (sets argtypes lazily)
    lib.paged_attn_decode_noalloc.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int] * 5 + [ctypes.c_float] + \
        [ctypes.c_int] * 2 + [ctypes.c_void_p] * 2
    rc = lib.paged_attn_decode_noalloc(P, P, P, P, P, P, 2048, 64, 8, 128, 16, 0.088, 256, 50000, None, None)
    msg = lib.pkv_last_error().decode()
    assert rc == -1 and "static scratch" in msg and str(SCRATCH_BYTES) in msg, msg
    need = pkv.workspace_bytes(2048, 64, 128)
    assert need > SCRATCH_BYTES and str(need) in msg
