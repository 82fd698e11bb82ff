"""Multi-query paged attention (chunked prefill, mixed batches) through the C
ABI, against the fp64 oracle: query i of a sequence's n-token chunk attends
causally to positions 0 .. L - n + i. Tolerance |err| <= 8e-3 + 8e-3 |ref|."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_377_b200 as pkv
import workloads
from helpers import assert_close_to_oracle, gather_contiguous, load_golden_prefill, prefill_golden_names

pytestmark = pytest.mark.gpu

DEV = "cuda"


def run(b, max_query_len=None, kernel=0):
    qs = b.query_start
    mq = int((qs[1:] - qs[:-1]).max()) if max_query_len is None else max_query_len
    out = torch.full(b.q.shape, float("nan"), dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    pkv.paged_attn_prefill(out, b.q.to(DEV), b.k_cache.to(DEV), b.v_cache.to(DEV), b.block_tables.to(DEV),
                           b.context_lens.to(DEV), qs.to(DEV), mq, b.scale, status, kernel=kernel)
    torch.cuda.synchronize()
    return out.cpu(), pkv.read_status(status)


def ref_of(b):
    return oracle.paged_prefill(b.q, b.k_cache, b.v_cache, b.block_tables.numpy(), b.context_lens.numpy(),
                                b.query_start.numpy(), b.num_kv_heads, b.block_size, b.scale)


@pytest.mark.parametrize("kernel", [1, 2])
@pytest.mark.parametrize("G", [1, 2, 4, 7, 8])
@pytest.mark.parametrize("D,bs", [(64, 16), (64, 32), (128, 16), (128, 32)])
def test_mixed_batch_matches_oracle(G, D, bs, kernel):
    chunks = [1, 7, 16, 64, 130, 0, 1, 33]
    ctx = [1, 40, 16, 64, 700, 9, 1029, 33]
    b = workloads.make_prefill(3000 + 11 * G + D + bs, chunks, ctx, 2 * G, 2, D, bs)
    if kernel == 2 and G not in (1, 2, 4, 8):
        with pytest.raises(pkv.PagedKVError, match="tcgen05"):
            run(b, kernel=2)
        return
    out, st = run(b, kernel=kernel)
    assert st == 0
    assert_close_to_oracle(out.double().numpy(), ref_of(b), what=f"prefill G={G} D={D} bs={bs} kernel={kernel}")


def test_single_token_chunks_match_the_decode_kernel():
    lens = [1, 5, 300, 1024, 77]
    b = workloads.make_prefill(3100, [1] * len(lens), lens, 32, 8, 128, 16)
    out, st = run(b)
    assert st == 0
    ref = ref_of(b)
    assert_close_to_oracle(out.double().numpy(), ref, what="n = 1")
    dec = torch.empty_like(b.q, device=DEV)
    ws = pkv.allocate_workspace(b.num_seqs, b.num_q_heads, b.head_dim, device=DEV)
    pkv.paged_attn_decode(dec, b.q.to(DEV), b.k_cache.to(DEV), b.v_cache.to(DEV), b.block_tables.to(DEV),
                          b.context_lens.to(DEV), b.scale, ws)
    assert_close_to_oracle(dec.double().cpu().numpy(), ref, what="decode kernel on the same rows")


@pytest.mark.parametrize("kernel", [1, 2])
def test_long_chunk_of_one_sequence(kernel):
    """One 300-token chunk at the end of a 2000-token context: several 128-row tiles, many iterations."""
    b = workloads.make_prefill(3150, [300, 4], [2000, 70], 16, 4, 128, 16)
    out, st = run(b, kernel=kernel)
    assert st == 0
    assert_close_to_oracle(out.double().numpy(), ref_of(b), what=f"long chunk kernel={kernel}")


@pytest.mark.parametrize("kernel", [1, 2])
@pytest.mark.parametrize("scale", [-0.2, 0.01, 1.5])
def test_scales_of_either_sign_and_size(kernel, scale):
    """A negative scale flips which logit is largest; a large one makes the running
    maximum move often (rescales of O in tensor memory)."""
    b = workloads.make_prefill(3160, [200, 9], [900, 300], 8, 2, 128, 16, scale=scale)
    out, st = run(b, kernel=kernel)
    assert st == 0
    assert_close_to_oracle(out.double().numpy(), ref_of(b), what=f"scale {scale} kernel={kernel}")


def test_long_tables_fall_back_to_the_mma_sync_kernel():
    """A block-table row too long for the tcgen05 kernel's shared memory: kernel 2
    refuses it, the default runs the mma.sync kernel."""
    b = workloads.make_prefill(3170, [20, 5], [90, 40], 8, 2, 128, 16)
    pad = torch.full((b.num_seqs, 40000 - b.block_tables.shape[1]), -1, dtype=torch.int32)
    b2 = workloads.PrefillBatch(**{**b.__dict__, "block_tables": torch.cat([b.block_tables, pad], dim=1)})
    with pytest.raises(pkv.PagedKVError, match="shared memory"):
        run(b2, kernel=2)
    out, st = run(b2)
    assert st == 0
    assert_close_to_oracle(out.double().numpy(), ref_of(b), what="long table, default kernel")


def _relayout(b, block_size, seed):
    """The same sequences in a fresh pool of block_size-token blocks, in a shuffled
    physical order; slots past each context hold NaN."""
    rows = gather_contiguous(b)
    nblk = [(int(L) + block_size - 1) // block_size for L in b.context_lens]
    NB = max(sum(nblk), 1)
    perm = np.random.default_rng(seed).permutation(NB)
    kc = torch.full((NB, block_size, b.num_kv_heads, b.head_dim), float("nan"), dtype=torch.float64)
    vc = kc.clone()
    tables = np.zeros((b.num_seqs, max(max(nblk), 1)), dtype=np.int32)
    nxt = 0
    for s_, (k, v) in enumerate(rows):
        for lb in range(nblk[s_]):
            p = int(perm[nxt])
            nxt += 1
            tables[s_, lb] = p
            t = np.arange(lb * block_size, min((lb + 1) * block_size, k.shape[0]))
            kc[p, :len(t)] = torch.from_numpy(k[t])
            vc[p, :len(t)] = torch.from_numpy(v[t])
    return workloads.PrefillBatch(**{**b.__dict__, "block_size": block_size, "num_blocks": NB,
                                     "max_blocks_per_seq": tables.shape[1], "block_tables": torch.from_numpy(tables),
                                     "k_cache": kc.to(torch.bfloat16), "v_cache": vc.to(torch.bfloat16)})


@pytest.mark.parametrize("kernel", [1, 2])
@pytest.mark.parametrize("bs", [16, 32])
@pytest.mark.parametrize("name", prefill_golden_names())
def test_worked_examples_give_their_exact_values(name, bs, kernel):
    """The multi-query golden fixtures (values derived by hand), re-laid in the
    kernels' block sizes: every output within the bf16 tolerance of its exact value."""
    b, expected = load_golden_prefill(name)
    out, st = run(_relayout(b, bs, seed=bs), kernel=kernel)
    assert st == 0
    got = out.double().numpy()
    for (r, j), row in expected.items():
        assert np.all(np.abs(got[r, j] - row) <= 8e-3 + 8e-3 * np.abs(row)), (name, r, j, got[r, j][:2], row[:2])


def test_llama_shaped_chunked_prefill_sampled_rows():
    rng = np.random.default_rng(31)
    chunks = [512, 256, 384, 128, 1, 1, 1, 1]
    ctx = [int(c + rng.integers(0, 3000)) for c in chunks]
    b = workloads.make_prefill(3200, chunks, ctx, 32, 8, 128, 16, device="cuda").to("cpu")
    out, st = run(b)
    assert st == 0
    T, Hq = b.q.shape[0], b.num_q_heads
    rows = np.random.default_rng(2).choice(T, size=48, replace=False)
    sub_qs = []
    # the oracle on the sampled query tokens only: one one-token chunk per sampled row
    qs = b.query_start.numpy()
    seq_of = np.searchsorted(qs, rows, side="right") - 1
    for r, s in zip(rows, seq_of):
        n = int(qs[s + 1] - qs[s])
        p = int(b.context_lens[s]) - n + int(r - qs[s])
        sub_qs.append((s, p + 1, r))
    lens = np.array([x[1] for x in sub_qs], dtype=np.int32)
    tables = b.block_tables.numpy()[[x[0] for x in sub_qs]]
    q = b.q[[x[2] for x in sub_qs]]
    ref = oracle.paged_decode(q, b.k_cache, b.v_cache, tables, lens, b.num_kv_heads, b.block_size, b.scale)
    assert_close_to_oracle(out[rows].double().numpy(), ref, what="llama-shaped chunked prefill (sampled)")


def test_inconsistent_chunks_are_flagged_and_skipped():
    b = workloads.make_prefill(3300, [3, 4], [10, 12], 4, 2, 64, 16)
    bad_lens = b.context_lens.clone()
    bad_lens[1] = 2                                   # a chunk of 4 cannot end a context of 2
    b2 = workloads.PrefillBatch(**{**b.__dict__, "context_lens": bad_lens})
    out, st = run(b2)
    assert st & pkv.PKV_STATUS_BAD_CONTEXT_LEN
    ref = ref_of(b)
    assert_close_to_oracle(out[:3].double().numpy(), ref[:3], what="the consistent sequence")


def test_bad_block_id_is_flagged_not_faulted():
    b = workloads.make_prefill(3400, [5, 2], [40, 20], 4, 2, 128, 16)
    tables = b.block_tables.clone()
    tables[0, 1] = b.num_blocks + 7
    b2 = workloads.PrefillBatch(**{**b.__dict__, "block_tables": tables})
    _, st = run(b2)
    assert st & pkv.PKV_STATUS_BAD_BLOCK_ID
