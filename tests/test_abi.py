"""The C-ABI library on a host without a GPU: it loads, exports every symbol the
header declares, and rejects bad arguments before any CUDA call."""
import ctypes
import os
import re

import numpy as np
import pytest

import paged_kv_cache_377_b200 as pkv

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "pagedkv.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)) - {"defined"})


def test_library_loads_and_exports_every_declared_symbol():
    lib = pkv.library()
    names = declared_functions()
    assert {"paged_attn_decode", "kv_cache_append", "pkv_decode_workspace_bytes"} <= set(names)
    for name in names:
        assert hasattr(lib, name), f"{name} declared in pagedkv.h but not exported"
    assert lib.pkv_version().startswith(b"pagedkv")


def test_workspace_size():
    # header | per-segment piece counters (<= S * Hq uint64, one launch of <= 2048 seqs)
    # | fp32 partials [rows][D] | fp32 log2-sum-exp [rows], rows = (S + 1024) * Hq
    def expect(S, Hq, D):
        sc = min(S, 2048)
        rows = (sc + 1024) * Hq
        return 256 + -(-sc * Hq * 8 // 256) * 256 + rows * D * 4 + -(-rows * 4 // 256) * 256
    for S, Hq, D in [(4, 2, 64), (256, 32, 128), (3000, 12, 64), (0, 8, 128)]:
        assert pkv.workspace_bytes(S, Hq, D) == expect(S, Hq, D)
    assert pkv.workspace_bytes(5000, 8, 128) == pkv.workspace_bytes(2048, 8, 128)
    with pytest.raises(pkv.PagedKVError, match="num_q_heads"):
        pkv.workspace_bytes(4, 0, 64)


P = ctypes.c_void_p(4096)  # a non-null, aligned address: argument checks never dereference it


def _decode(**kw):
    args = dict(out=P, q=P, k=P, v=P, bt=P, cl=P, S=4, Hq=2, Hkv=1, D=64, bs=16, scale=0.125, MB=3, NB=16,
                ws=P, wsb=1 << 20)
    args.update(kw)
    lib = pkv.library()
    rc = lib.paged_attn_decode(args["out"], args["q"], args["k"], args["v"], args["bt"], args["cl"], args["S"],
                               args["Hq"], args["Hkv"], args["D"], args["bs"], args["scale"], args["MB"],
                               args["NB"], args["ws"], args["wsb"], None)
    return rc, lib.pkv_last_error().decode()


@pytest.mark.parametrize("kw,code,msg", [
    (dict(q=None), -1, "NULL"),
    (dict(ws=None), -1, "NULL"),
    (dict(S=-1), -1, "num_seqs"),
    (dict(Hq=3, Hkv=2), -1, "multiple"),
    (dict(D=96), -2, "head_dim"),
    (dict(bs=8), -2, "block_size"),
    (dict(Hq=16, Hkv=1), -2, "exceeds"),
    (dict(scale=float("inf")), -1, "scale"),
    (dict(q=ctypes.c_void_p(4098)), -1, "aligned"),
    (dict(wsb=16), -1, "workspace_bytes"),
    (dict(Hkv=2, Hq=2, MB=1 << 20), -1, "too large"),
    (dict(NB=1 << 28), -1, "2^31"),
])
def test_decode_rejects_bad_arguments_without_touching_the_gpu(kw, code, msg):
    rc, err = _decode(**kw)
    assert rc == code and msg in err, (rc, err)


def test_decode_of_empty_batch_is_a_no_op():
    rc, err = _decode(S=0)
    assert rc == 0, err


def test_append_rejects_bad_arguments():
    lib = pkv.library()
    rc = lib.kv_cache_append(P, P, P, P, P, 4, 1, 60, 16, 16, None, None)
    assert rc == -2 and "multiple of 8" in lib.pkv_last_error().decode()
    rc = lib.kv_cache_append(P, None, P, P, P, 4, 1, 64, 16, 16, None, None)
    assert rc == -1
    rc = lib.kv_cache_append(P, P, P, P, P, 0, 1, 64, 16, 16, None, None)
    assert rc == 0


def test_options_are_checked():
    lib = pkv.library()
    opts = pkv._binding._Options(2000, 0, 0, 0, 0, 0)
    rc = lib.paged_attn_decode_ex(P, P, P, P, P, P, 4, 2, 1, 64, 16, 0.125, 3, 16, P, 1 << 20,
                                  ctypes.byref(opts), None)
    assert rc == -1 and "num_ctas" in lib.pkv_last_error().decode()
    opts = pkv._binding._Options(0, 5, 0, 0, 0, 0)
    rc = lib.paged_attn_decode_ex(P, P, P, P, P, P, 4, 2, 1, 64, 16, 0.125, 3, 16, P, 1 << 20,
                                  ctypes.byref(opts), None)
    assert rc == -1 and "num_stages" in lib.pkv_last_error().decode()
    opts = pkv._binding._Options(0, 0, 0, 0, 0, 0, 3)
    rc = lib.paged_attn_decode_ex(P, P, P, P, P, P, 4, 2, 1, 64, 16, 0.125, 3, 16, P, 1 << 20,
                                  ctypes.byref(opts), None)
    assert rc == -1 and "unknown option" in lib.pkv_last_error().decode()
    # packing two kv heads needs an even number of them (here 1) and head_dim 64
    opts = pkv._binding._Options(0, 0, 0, 0, 0, 0, 2)
    rc = lib.paged_attn_decode_ex(P, P, P, P, P, P, 4, 2, 1, 64, 16, 0.125, 3, 16, P, 1 << 20,
                                  ctypes.byref(opts), None)
    assert rc == -2 and "head_pack" in lib.pkv_last_error().decode()
    rc = lib.paged_attn_decode_ex(P, P, P, P, P, P, 4, 8, 2, 128, 16, 0.125, 3, 16, P, 1 << 20,
                                  ctypes.byref(opts), None)
    assert rc == -2 and "head_pack" in lib.pkv_last_error().decode()
    # tiles of 16 or 32 token rows, never more than a block
    opts = pkv._binding._Options(0, 0, 0, 0, 0, 0, 0, 24)
    rc = lib.paged_attn_decode_ex(P, P, P, P, P, P, 4, 2, 1, 64, 32, 0.125, 3, 16, P, 1 << 20,
                                  ctypes.byref(opts), None)
    assert rc == -1 and "unknown option" in lib.pkv_last_error().decode()
    opts = pkv._binding._Options(0, 0, 0, 0, 0, 0, 0, 32)
    rc = lib.paged_attn_decode_ex(P, P, P, P, P, P, 4, 2, 1, 64, 16, 0.125, 3, 16, P, 1 << 20,
                                  ctypes.byref(opts), None)
    assert rc == -1 and "tile_tokens" in lib.pkv_last_error().decode()


def test_fused_step_checks_its_extra_arguments():
    lib = pkv.library()
    args = [P, P, P, P, P, P, P, P, P, 4, 2, 1, 64, 16, 0.125, 3, 16, P, 1 << 20, None, None]
    bad = list(args)
    bad[4] = None  # slot_mapping
    assert lib.paged_attn_decode_append(*bad) == -1 and "slot_mapping" in lib.pkv_last_error().decode()
    bad = list(args)
    bad[2] = None  # k_new
    assert lib.paged_attn_decode_append(*bad) == -1 and "k_new" in lib.pkv_last_error().decode()
    bad = list(args)
    bad[3] = ctypes.c_void_p(4096 + 8)  # v_new misaligned
    assert lib.paged_attn_decode_append(*bad) == -1 and "aligned" in lib.pkv_last_error().decode()


def test_block_copy_checks_arguments():
    lib = pkv.library()
    pkv.block_manager._lib()  # sets the argument types
    assert lib.kv_block_copy(P, P, None, P, 2, 2, 64, 2, 16, 8, None, None) == -1
    assert "NULL" in lib.pkv_last_error().decode()
    assert lib.kv_block_copy(P, P, P, P, 2, 2, 60, 2, 16, 8, None, None) == -2
    assert lib.kv_block_copy(P, P, P, P, 2, 2, 24, 1, 16, 8, None, None) == -2   # 24-byte rows
    assert lib.kv_block_copy(P, P, P, P, 2, 2, 64, 4, 16, 8, None, None) == -1   # elem_bytes
    assert lib.kv_block_copy(P, P, P, P, -1, 2, 64, 2, 16, 8, None, None) == -1
    assert lib.kv_block_copy(P, P, None, None, 0, 2, 64, 2, 16, 8, None, None) == 0  # nothing to copy


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        pkv.paged_attn_decode(q, q, q[None], q[None], torch.zeros(1, 1, dtype=torch.int32),
                              torch.zeros(1, dtype=torch.int32), 0.1, torch.zeros(256, dtype=torch.uint8))


def test_missing_library_fails_loudly(monkeypatch):
    """No CPU fallback: when the library can be neither found nor built, calls raise."""
    from paged_kv_cache_377_b200 import _binding

    def no_build(*a, **k):
        raise RuntimeError("nvcc not found")

    monkeypatch.setattr(_binding, "_lib", None)
    monkeypatch.setattr(_binding._build, "is_stale", lambda: True)
    monkeypatch.setattr(_binding._build, "build", no_build)
    with pytest.raises(RuntimeError, match="nvcc"):
        pkv.workspace_bytes(1, 1, 64)


def _prefill(**kw):
    args = dict(out=P, q=P, k=P, v=P, bt=P, cl=P, qs=P, S=2, T=9, MQ=5, Hq=8, Hkv=2, D=128, bs=16, scale=0.125,
                MB=8, NB=32, st=P, kernel=0)
    args.update(kw)
    lib = pkv.library()
    rc = lib.paged_attn_prefill_ex(args["out"], args["q"], args["k"], args["v"], args["bt"], args["cl"], args["qs"],
                                   args["S"], args["T"], args["MQ"], args["Hq"], args["Hkv"], args["D"], args["bs"],
                                   args["scale"], args["MB"], args["NB"], args["st"], args["kernel"], None)
    return rc, lib.pkv_last_error().decode()


@pytest.mark.parametrize("kw,code,msg", [
    (dict(kernel=3), -1, "kernel must be"),
    (dict(st=None), -1, "NULL"),
    (dict(qs=None), -1, "NULL"),
    (dict(MQ=-1), -1, "max_query_len"),
    (dict(Hq=6, Hkv=4), -1, "multiple"),
    (dict(D=96), -2, "head_dim"),
    (dict(bs=8), -2, "block_size"),
    (dict(Hq=32, Hkv=2), -2, "exceeds"),
    (dict(scale=float("nan")), -1, "scale"),
    (dict(out=ctypes.c_void_p(4096 + 8)), -1, "aligned"),
    (dict(kernel=2, Hq=6, Hkv=2), -2, "tcgen05"),                       # group 3: 128 rows are not whole tokens
    (dict(kernel=2, MB=40000), -2, "shared memory"),                   # the table row does not fit beside the tiles
])
def test_prefill_rejects_bad_arguments_without_touching_the_gpu(kw, code, msg):
    rc, err = _prefill(**kw)
    assert rc == code and msg in err, (rc, err)


@pytest.mark.parametrize("kw", [dict(S=0), dict(T=0), dict(MQ=0), dict(T=0, kernel=2), dict(T=0, kernel=1)])
def test_prefill_of_empty_batch_is_a_no_op(kw):
    rc, err = _prefill(**kw)
    assert rc == 0, err


@pytest.mark.parametrize("bad", ["out", "v_cache", "head_dim", "block_tables", "context_lens"])
def test_noalloc_binding_checks_shapes_before_calling_the_library(monkeypatch, bad):
    """paged_attn_decode_noalloc's binding checks that the tensors agree, like
    paged_attn_decode's: the C ABI cannot see tensor lengths, so a short table or
    a head_dim mismatch would reach the kernel as out-of-bounds accesses."""
    import torch
    from paged_kv_cache_377_b200 import _binding

    calls = []
    monkeypatch.setattr(_binding, "_need", lambda *a, **k: None)      # CPU tensors stand in for device ones
    monkeypatch.setattr(_binding, "library", lambda: calls.append(1))
    S, Hq, Hkv, D, NB, bs, MB = 3, 8, 2, 64, 10, 16, 4
    t = dict(out=torch.zeros(S, Hq, D, dtype=torch.bfloat16), q=torch.zeros(S, Hq, D, dtype=torch.bfloat16),
             k_cache=torch.zeros(NB, bs, Hkv, D, dtype=torch.bfloat16),
             v_cache=torch.zeros(NB, bs, Hkv, D, dtype=torch.bfloat16),
             block_tables=torch.zeros(S, MB, dtype=torch.int32), context_lens=torch.zeros(S, dtype=torch.int32))
    if bad == "out":
        t["out"] = torch.zeros(S + 1, Hq, D, dtype=torch.bfloat16)
    elif bad == "v_cache":
        t["v_cache"] = torch.zeros(NB - 1, bs, Hkv, D, dtype=torch.bfloat16)
    elif bad == "head_dim":
        t["k_cache"] = t["v_cache"] = torch.zeros(NB, bs, Hkv, 2 * D, dtype=torch.bfloat16)
    elif bad == "block_tables":
        t["block_tables"] = torch.zeros(S - 1, MB, dtype=torch.int32)
    else:
        t["context_lens"] = torch.zeros(S - 1, dtype=torch.int32)
    with pytest.raises(ValueError):
        _binding.paged_attn_decode_noalloc(t["out"], t["q"], t["k_cache"], t["v_cache"], t["block_tables"],
                                           t["context_lens"], 0.125)
    assert calls == [], "the library was reached with inconsistent shapes"


def test_find_prefix_groups_on_host_tables():
    bt = np.array([[5, 6, 7, -1], [5, 6, 9, -1], [5, 6, 7, 8], [1, 2, 3, -1], [1, 2, 4, -1], [0, -1, -1, -1],
                   [3, 4, -1, -1], [3, 4, -1, -1]], dtype=np.int32)
    cl = np.array([40, 35, 60, 33, 33, 10, 20, 32], dtype=np.int32)
    g = pkv.find_prefix_groups(bt, cl, 16)
    assert g.begin.tolist() == [0, 3, 6] and g.end.tolist() == [3, 5, 8] and g.blocks.tolist() == [2, 2, 2]
    # a context that covers fewer entries bounds what the run shares (seq 6 covers 2 blocks)
    g = pkv.find_prefix_groups(bt[6:], cl[6:], 16)
    assert g.blocks.tolist() == [2]
    assert len(pkv.find_prefix_groups(bt, cl, 16, min_blocks=3)) == 0
    assert len(pkv.find_prefix_groups(bt, cl, 16, max_groups=2)) == 2
    lib = pkv.library()
    n = ctypes.c_int(0)
    assert lib.pkv_find_prefix_groups(None, None, 3, 4, 16, 1, None, None, None, 0, ctypes.byref(n)) == -1
    assert lib.pkv_find_prefix_groups(None, None, 0, 4, 16, 1, None, None, None, 0, ctypes.byref(n)) == 0 and n.value == 0


@pytest.mark.parametrize("begin,end,blocks,code,msg", [
    ([0], [1], [2], -1, "two or more"),
    ([2, 3], [4, 5], [2, 2], -1, "two or more"),       # overlapping groups
    ([0], [5], [2], -1, "two or more"),                # past num_seqs (4)
    ([0], [3], [0], -1, "blocks"),
    ([0], [3], [4], -1, "blocks"),                     # more than max_blocks_per_seq (3)
])
def test_decode_checks_prefix_groups_without_touching_the_gpu(begin, end, blocks, code, msg):
    lib = pkv.library()
    groups = pkv.PrefixGroups(begin, end, blocks)
    opts = pkv._binding._options(prefix_groups=groups)
    rc = lib.paged_attn_decode_ex(P, P, P, P, P, P, 4, 2, 1, 64, 16, 0.125, 3, 16, P, 1 << 20,
                                  ctypes.byref(opts), None)
    assert rc == code and msg in lib.pkv_last_error().decode(), (rc, lib.pkv_last_error())


def test_prefix_groups_need_bf16_pools_on_tensor_cores():
    lib = pkv.library()
    groups = pkv.PrefixGroups([0], [3], [2])
    for kw, msg in [(dict(math=1), "tensor cores"), (dict(head_pack=2), "head packing"), (dict(tile_tokens=32), "16-row")]:
        opts = pkv._binding._options(prefix_groups=groups, **kw)
        rc = lib.paged_attn_decode_ex(P, P, P, P, P, P, 4, 4, 2, 64, 32, 0.125, 3, 16, P, 1 << 20,
                                      ctypes.byref(opts), None)
        assert rc == -2 and msg in lib.pkv_last_error().decode(), (kw, rc, lib.pkv_last_error())
    opts = pkv._binding._options(prefix_groups=groups)
    rc = lib.paged_attn_decode_fp8(P, P, P, P, P, P, P, P, 4, 4, 2, 128, 16, 0.125, 3, 16, P, 1 << 20,
                                   ctypes.byref(opts), None)
    assert rc == -2 and "tensor cores" in lib.pkv_last_error().decode()


def test_prepared_decode_call_checks_its_tensors_once_at_construction():
    """DecodeAppendCall runs the fused step's argument checks when built (here:
    host tensors are refused before anything is enqueued)."""
    import torch
    S, Hq, Hkv, D, NB, bs = 2, 4, 2, 64, 8, 16
    bf = torch.bfloat16
    args = (torch.empty(S, Hq, D, dtype=bf), torch.empty(S, Hq, D, dtype=bf), torch.empty(S, Hkv, D, dtype=bf),
            torch.empty(S, Hkv, D, dtype=bf), torch.zeros(S, dtype=torch.int64), torch.empty(NB, bs, Hkv, D, dtype=bf),
            torch.empty(NB, bs, Hkv, D, dtype=bf), torch.zeros(S, 4, dtype=torch.int32),
            torch.ones(S, dtype=torch.int32), 0.125, torch.zeros(1 << 16, dtype=torch.uint8))
    with pytest.raises(ValueError, match="CUDA device"):
        pkv.DecodeAppendCall(*args)


def test_prepared_fp8_call_checks_its_tensors_once_at_construction():
    """DecodeAppendFp8Call runs the e4m3 fused step's argument checks when built
    (host tensors are refused before anything is enqueued)."""
    import torch
    S, Hq, Hkv, D, NB, bs = 2, 4, 2, 128, 8, 16
    bf, u8 = torch.bfloat16, torch.uint8
    good = [torch.empty(S, Hq, D, dtype=bf), torch.empty(S, Hq, D, dtype=bf), torch.empty(S, Hkv, D, dtype=bf),
            torch.empty(S, Hkv, D, dtype=bf), torch.zeros(S, dtype=torch.int64), torch.empty(NB, bs, Hkv, D, dtype=u8),
            torch.empty(NB, bs, Hkv, D, dtype=u8), torch.ones(Hkv), torch.ones(Hkv), torch.zeros(S, 4, dtype=torch.int32),
            torch.ones(S, dtype=torch.int32), 0.125, torch.zeros(1 << 16, dtype=u8)]
    with pytest.raises(ValueError, match="CUDA device"):
        pkv.DecodeAppendFp8Call(*good)
