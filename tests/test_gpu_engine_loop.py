"""Several continuous-batching iterations driven by the native block manager, on the GPU.

Per iteration, as the pages describe an engine step (vLLM overview, "Continuous Batching" and
"Prefix Sharing"; Core Concepts §3.2):
- requests join (their prompt is appended and attended by the causal prefill);
- running requests decode one token each (append at the end of the current block, new block when
  full, copy-on-write when the block is shared after a fork);
- a request forks for parallel sampling;
- a finished request leaves and its blocks are reused.
Every attention output is checked against the oracle, computed from each request's own token history
in a fresh contiguous cache.
"""
import numpy as np
import pytest
import torch

from pagedattention_block_table_b200.inputs import bf16_bits
from tests.common import assert_close, to_f64

pytestmark = pytest.mark.gpu

HQ, HKV, D = 8, 2, 128
SCALE = D ** -0.5


def _oracle_rows(O, k_rows, v_rows, q_rows, lens):
    """Attention of q_rows[i] over the first lens[i] tokens of (k_rows, v_rows), contiguous cache."""
    L = k_rows.shape[0]
    nblk = (L + 15) // 16
    kc = np.zeros((nblk, HKV, 16, D), np.uint16)
    vc = np.zeros_like(kc)
    O.kv_append(kc, vc, k_rows, v_rows, np.arange(L, dtype=np.int64))
    n = q_rows.shape[0]
    tables = np.tile(np.arange(nblk, dtype=np.int32)[None], (n, 1))
    return O.paged_decode(q_rows, kc, vc, tables, np.asarray(lens, np.int32), SCALE)


@pytest.mark.parametrize("bs", [16, 32])
def test_block_manager_drives_append_prefill_decode(O, cuda_lib, bs):
    B = cuda_lib
    g = torch.Generator(device="cuda").manual_seed(7)
    nb = 256 * 16 // bs
    kc = torch.zeros((nb, HKV, bs, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    bm = B.pa_bm_create(nb, bs, 99)
    hist = {}                                   # request id -> (K rows, V rows) on the device

    def new_tokens(n):
        return (torch.randn((n, HKV, D), generator=g, device="cuda").to(torch.bfloat16),
                torch.randn((n, HKV, D), generator=g, device="cuda").to(torch.bfloat16))

    def append(rid, k, v):
        slots, cow = B.pa_bm_append(bm, rid, k.shape[0])
        if cow is not None:
            B.pa_copy_blocks(kc, vc, torch.from_numpy(cow.reshape(1, 2)).cuda())
        B.pa_kv_append(kc, vc, k, v, torch.from_numpy(slots).cuda())
        hk, hv = hist.get(rid, (k[:0], v[:0]))
        hist[rid] = (torch.cat([hk, k]), torch.cat([hv, v]))
        return cow

    def prefill(rids, chunks):
        """Causal prefill of the chunks just appended to requests `rids`."""
        lens = [B.pa_bm_length(bm, r) for r in rids]
        mbs = max((L + bs - 1) // bs for L in lens)
        tables, tl = B.pa_bm_tables(bm, rids, mbs)
        cu = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
        q = torch.randn((int(cu[-1]), HQ, D), generator=g, device="cuda").to(torch.bfloat16)
        out = torch.empty_like(q)
        B.pa_paged_prefill(out, q, torch.from_numpy(cu).cuda(), kc, vc, torch.from_numpy(tables).cuda(),
                           torch.from_numpy(tl).cuda(), SCALE, max(chunks), max(lens))
        torch.cuda.synchronize()
        got = to_f64(out)
        for i, r in enumerate(rids):
            C, L = chunks[i], lens[i]
            k, v = hist[r]
            qb = bf16_bits(q[cu[i]:cu[i + 1]])
            ref = _oracle_rows(O, bf16_bits(k), bf16_bits(v), qb, [L - C + j + 1 for j in range(C)])
            assert_close(got[cu[i]:cu[i + 1]], ref, what=f"prefill of request {r}")

    def decode(rids):
        lens = [B.pa_bm_length(bm, r) for r in rids]
        mbs = max((L + bs - 1) // bs for L in lens)
        tables, tl = B.pa_bm_tables(bm, rids, mbs)
        q = torch.randn((len(rids), HQ, D), generator=g, device="cuda").to(torch.bfloat16)
        out = torch.empty_like(q)
        ws = torch.empty(B.pa_paged_attention_workspace_size(len(rids), HQ, D, max(lens), 64) // 4 + 4,
                         device="cuda")
        B.pa_paged_attention(out, q, kc, vc, torch.from_numpy(tables).cuda(), torch.from_numpy(tl).cuda(), SCALE,
                             max(lens), split_tokens=64, workspace=ws)
        torch.cuda.synchronize()
        got = to_f64(out)
        for i, r in enumerate(rids):
            k, v = hist[r]
            ref = _oracle_rows(O, bf16_bits(k), bf16_bits(v), bf16_bits(q[i:i + 1]), [lens[i]])
            assert_close(got[i], ref[0], what=f"decode of request {r}")

    try:
        # iteration 1: two requests join with prompts of 37 and 100 tokens
        for rid, n in ((1, 37), (2, 100)):
            B.pa_bm_add(bm, rid)
            append(rid, *new_tokens(n))
        prefill([1, 2], [37, 100])
        cows = 0
        for it in range(6):
            if it == 2:                          # request 1 forks (parallel sampling): shares every page
                B.pa_bm_fork(bm, 1, 3)
                hist[3] = hist[1]
            if it == 4:                          # request 2 finishes and leaves; request 4 joins
                B.pa_bm_free(bm, 2)
                del hist[2]
                B.pa_bm_add(bm, 4)
                append(4, *new_tokens(50))
                prefill([4], [50])
            running = sorted(hist)
            for r in running:
                cows += append(r, *new_tokens(1)) is not None
            decode(running)
        assert cows >= 1, "the fork must have triggered copy-on-write"
        assert B.pa_get_device_error() == B.PA_OK
    finally:
        B.pa_bm_destroy(bm)


def test_cuda_graph_replay_matches_eager(cuda_lib):
    """A serving step captured in a CUDA graph (the library's launches keep their programmatic
    dependencies inside the graph) and replayed gives bit-identical outputs to the eager step.
    The step is the mixed one without forks, so that repeating it is idempotent."""
    from pagedattention_block_table_b200.inputs import make_batch
    from pagedattention_block_table_b200.runner import DeviceStep
    small = dict(num_seqs=6, hist=("uniform", 100, 2500), share_group=0, share_prefix=0, num_q_heads=8,
                 num_kv_heads=2, head_dim=128, prefill_chunks=2, chunk_len=(40, 300), chunk_hist=(1, 600))
    st = DeviceStep(make_batch("mixed_step", seed=81, overrides=small), split_tokens=256)
    st.fill_history()
    st.step()
    torch.cuda.synchronize()
    eager_dec, eager_pre = st.out_dec.clone(), st.out_pre.clone()
    st.out_dec.zero_()
    st.out_pre.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=torch.cuda.Stream()):
        st.step()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert cuda_lib.pa_get_device_error() == cuda_lib.PA_OK
    assert torch.equal(st.out_dec, eager_dec)
    assert torch.equal(st.out_pre, eager_pre)


def test_prefix_tree_shared_blocks_feed_the_kernels(O, cuda_lib):
    """Two prompts with a common 40-token start: the second shares the first's two full blocks through
    the block manager's prefix tree (once the first has committed them), appends K/V only for its own
    tokens, and
    - its causal prefill over the whole prompt (read through the shared blocks), and
    - the prefill of only its new rows as one chunk whose history is the shared part (H = reused, the
      flow a serving engine runs)
    match the oracle on its own contiguous K/V."""
    B = cuda_lib
    g = torch.Generator(device="cuda").manual_seed(11)
    nb = 64
    kc = torch.zeros((nb, HKV, 16, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    rnd = lambda n: torch.randn((n, HKV, D), generator=g, device="cuda").to(torch.bfloat16)
    common_k, common_v = rnd(40), rnd(40)        # K/V of the common start (same tokens, same positions)
    rng = np.random.default_rng(2)
    common = rng.integers(0, 32000, 40)
    p1 = np.concatenate([common, rng.integers(0, 32000, 25)])
    p2 = np.concatenate([common, rng.integers(0, 32000, 57)])
    k1 = torch.cat([common_k, rnd(25)])
    v1 = torch.cat([common_v, rnd(25)])
    k2 = torch.cat([common_k, rnd(57)])
    v2 = torch.cat([common_v, rnd(57)])
    bm = B.pa_bm_create(nb, 16, 4)
    try:
        s1, r1 = B.pa_bm_add_prompt(bm, 1, p1)
        B.pa_kv_append(kc, vc, k1, v1, torch.from_numpy(s1).cuda())
        B.pa_bm_commit(bm, 1, len(p1))
        s2, r2 = B.pa_bm_add_prompt(bm, 2, p2)
        assert r1 == 0 and r2 == 32
        B.pa_kv_append(kc, vc, k2[r2:].contiguous(), v2[r2:].contiguous(), torch.from_numpy(s2).cuda())
        B.pa_bm_commit(bm, 2, len(p2))
        n = len(p2)
        tables, tl = B.pa_bm_tables(bm, [2], (n + 15) // 16)
        q = torch.randn((n, HQ, D), generator=g, device="cuda").to(torch.bfloat16)
        ref = _oracle_rows(O, bf16_bits(k2), bf16_bits(v2), bf16_bits(q), [i + 1 for i in range(n)])
        # the whole prompt as one chunk (H = 0)
        out = torch.empty_like(q)
        cu = torch.tensor([0, n], dtype=torch.int32, device="cuda")
        B.pa_paged_prefill(out, q, cu, kc, vc, torch.from_numpy(tables).cuda(), torch.from_numpy(tl).cuda(),
                           SCALE, n, n)
        # only the new rows r2 .. n-1, as one chunk over the shared history (H = r2)
        qn = q[r2:].contiguous()
        outn = torch.empty_like(qn)
        cun = torch.tensor([0, n - r2], dtype=torch.int32, device="cuda")
        B.pa_paged_prefill(outn, qn, cun, kc, vc, torch.from_numpy(tables).cuda(), torch.from_numpy(tl).cuda(),
                           SCALE, n - r2, n)
        torch.cuda.synchronize()
        assert B.pa_get_device_error() == B.PA_OK
        assert_close(to_f64(out), ref, what="prefill over prefix-shared blocks")
        assert_close(to_f64(outn), ref[r2:], what="new rows over the shared history")
    finally:
        B.pa_bm_destroy(bm)
