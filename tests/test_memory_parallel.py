"""Memory Parallel (the memory's documents split over GPUs, each routing its own part, the
results reduced to one global top-k: Evermind summary sec. 4B; b-lab.team item 2).

CPU: the document partition, and the host logic of the exchange over two gloo ranks -- each rank
routes its shard (the oracle stands in for the CUDA route on the CPU), the candidates are
all-gathered, and their merge is the global top-k of the whole memory.
GPU (one device, 2 and 4 logical shards): the shards' msa_route candidates merged by
msa_topk_merge are bit-identical to msa_route over the whole memory, and to the oracle's top-k of
the concatenated state; exact ties across shard boundaries go to the lower global id."""
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from top_document_sparse_b200 import inputs
from top_document_sparse_b200.memory_parallel import (gather_candidates, shard_ranges,
                                                      shard_token_offsets)

from helpers import memory_inputs, small_workload

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("n_shards", [1, 2, 3, 7])
def test_shard_ranges_cover_the_documents_in_balanced_contiguous_ranges(n_shards):
    w = small_workload(n_docs=0, doc_len=0, lognormal=(150, 1.0, 5, 900, 20000))
    off = inputs.doc_offsets(w, 4)
    b = shard_ranges(off, n_shards)
    assert b[0] == 0 and b[-1] == off.size - 1 and np.all(np.diff(b) >= 1)
    tok = np.diff(off[b])
    # each cut is at the first document boundary at or past its share of the tokens
    longest = int(np.max(np.diff(off)))
    assert np.all(np.abs(tok - off[-1] / n_shards) <= longest)
    sub = shard_token_offsets(off, b[1 % n_shards], b[1 % n_shards + 1])
    assert sub[0] == 0 and np.array_equal(np.diff(sub), np.diff(off)[b[1 % n_shards]:
                                                                     b[1 % n_shards + 1]])


def test_shard_ranges_rejects_more_shards_than_documents():
    with pytest.raises(ValueError):
        shard_ranges(np.array([0, 5, 9]), 3)


def _gloo_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle as orc
    from helpers import memory_inputs as mi, small_workload as sw
    from top_document_sparse_b200.memory_parallel import (gather_candidates as gc,
                                                          shard_ranges as sr,
                                                          shard_token_offsets as sto)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = sw(dtype="f32", n_docs=0, doc_len=0, lognormal=(120, 1.0, 5, 600, 8000), batch=3,
               query_tokens=5, top_k=4, head_dim=64, planted_per_query=2)
        inp = mi(w, seed=70)
        off = inp["off"]
        b = sr(off, world)
        d0, d1 = int(b[rank]), int(b[rank + 1])
        t0, t1 = int(off[d0]), int(off[d1])
        sub = sto(off, d0, d1)
        # this rank's shard: encode and route its own documents only
        _, _, Krb = orc.encode(inp["K"][t0:t1], inp["V"][t0:t1], inp["Kr"][t0:t1], sub,
                               w.chunk_len, w.rope_theta)
        st = orc.route(inp["Qr"], Krb, orc.doc_chunks(sub, w.chunk_len))
        ids, sc = orc.topk(st, w.top_k)
        # (the oracle's scores travel in fp64: two planted documents 1e-16 apart would tie in
        # fp32; the GPU path carries its own fp32 scores)
        scores_all, ids_all = gc(torch.from_numpy(sc), torch.from_numpy(ids), None)
        q.put((rank, d0, d1, scores_all.numpy(), ids_all.numpy(), b))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_candidate_exchange_over_gloo_gives_the_global_top_k():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29600 + os.getpid() % 1000
    procs = [ctx.Process(target=_gloo_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    # both ranks hold the same gathered candidates, in rank order
    assert np.array_equal(res[0][3], res[1][3]) and np.array_equal(res[0][4], res[1][4])
    scores_all, ids_all, bounds = res[0][3], res[0][4], res[0][5]
    # the whole memory, routed at once by the oracle
    w = small_workload(dtype="f32", n_docs=0, doc_len=0, lognormal=(120, 1.0, 5, 600, 8000),
                       batch=3, query_tokens=5, top_k=4, head_dim=64, planted_per_query=2)
    inp = memory_inputs(w, seed=70)
    _, _, Krb = oracle.encode(inp["K"], inp["V"], inp["Kr"], inp["off"], w.chunk_len,
                              w.rope_theta)
    full = oracle.route(inp["Qr"], Krb, oracle.doc_chunks(inp["off"], w.chunk_len))
    want_ids, want_sc = oracle.topk(full, w.top_k)
    # merge: the candidates at their global ids, ranked by (score desc, id asc)
    merged = np.full(full.shape, -np.inf)
    for s in range(2):
        for bq in range(3):
            for r in range(w.top_k):
                merged[bq, bounds[s] + ids_all[s, bq, r]] = scores_all[s, bq, r]
    got_ids, got_sc = oracle.topk(merged, w.top_k)
    assert np.array_equal(got_ids, want_ids)
    assert np.array_equal(got_sc, want_sc)


# ------------------------------------------------------------------------------------ GPU
def _shards(w, inp, n_shards, max_local=64):
    from top_document_sparse_b200.memory_parallel import MemoryShard
    b = shard_ranges(inp["off"], n_shards)
    dt = inputs.torch_dtype(w.dtype)
    K, V, Kr = (inp[n].cuda() for n in ("K", "V", "Kr"))
    out = []
    for s in range(n_shards):
        sh = MemoryShard(inp["off"], b, s, w.chunk_len, w.n_kv_heads, w.head_dim,
                         w.n_router_heads, w.router_dim, dt, w.rope_theta, max_local)
        rk, ct = sh.mem.new_router_keys(), sh.mem.new_content()
        sh.encode(K, V, Kr, rk, ct)
        out.append((sh, rk, ct))
    torch.cuda.synchronize()
    return b, out


@pytest.mark.gpu
@pytest.mark.parametrize("n_shards", [2, 4])
def test_merged_shard_top_k_is_bit_identical_to_the_whole_memory(n_shards):
    from top_document_sparse_b200 import msa
    w = small_workload(n_docs=0, doc_len=0, lognormal=(200, 1.0, 5, 1500, 60000), batch=6,
                       query_tokens=9, top_k=16, planted_per_query=5)
    inp = memory_inputs(w, seed=71)
    B, T, k = w.batch, w.query_tokens, w.top_k
    Qr = inp["Qr"].cuda()
    # the whole memory
    mem = msa.Memory(inp["off"], w.chunk_len, w.n_kv_heads, w.head_dim, w.n_router_heads,
                     w.router_dim, torch.bfloat16, w.rope_theta, 64)
    rk, ct = mem.new_router_keys(), mem.new_content()
    mem.encode(0, mem.n_docs, inp["K"].cuda(), inp["V"].cuda(), inp["Kr"].cuda(), rk, ct)
    state = torch.full((B, mem.n_docs), float("-inf"), device="cuda")
    ids = torch.zeros(B, k, dtype=torch.int32, device="cuda")
    scores = torch.zeros(B, k, device="cuda")
    mem.route(rk, Qr, k, state, ids, scores, msa.workspace(mem.route_workspace_size(B, T, k)))
    # the shards, each routing its own documents
    bounds, shards = _shards(w, inp, n_shards)
    c_sc = torch.empty(n_shards, B, k, device="cuda")
    c_id = torch.empty(n_shards, B, k, dtype=torch.int32, device="cuda")
    st_shard = []
    for s, (sh, srk, _) in enumerate(shards):
        st = torch.full((B, sh.mem.n_docs), float("-inf"), device="cuda")
        sh.route(srk, Qr, k, st, c_id[s], c_sc[s],
                 msa.workspace(sh.mem.route_workspace_size(B, T, k)))
        st_shard.append(st)
    g_ids, g_sc = msa.topk_merge(c_sc, c_id, bounds[:-1], k)
    torch.cuda.synchronize()
    # a document's score does not depend on the partition
    assert torch.equal(torch.cat(st_shard, dim=1), state)
    assert torch.equal(g_ids, ids) and torch.equal(g_sc, scores)
    want_ids, want_sc = oracle.topk(state.cpu().numpy().astype(np.float64), k)
    assert np.array_equal(g_ids.cpu().numpy(), want_ids)
    assert np.array_equal(g_sc.cpu().numpy().astype(np.float64), want_sc)
    assert msa.device_error() == 0


@pytest.mark.gpu
def test_merge_breaks_exact_ties_across_shards_by_global_id():
    """States with many exact ties, some straddling shard boundaries: the merge of the shards'
    top-k is the oracle's top-k of the whole state, id for id."""
    from top_document_sparse_b200 import msa
    B, n_docs, k = 4, 3000, 24
    rng = np.random.default_rng(9)
    full = (rng.integers(-8, 8, size=(B, n_docs)) / 8.0).astype(np.float32)
    bounds = np.array([0, 700, 701, 1999, n_docs])  # one shard of a single document
    n_shards = bounds.size - 1
    c_sc = torch.empty(n_shards, B, k, device="cuda")
    c_id = torch.empty(n_shards, B, k, dtype=torch.int32, device="cuda")
    for s in range(n_shards):
        nd = int(bounds[s + 1] - bounds[s])
        off = np.arange(nd + 1, dtype=np.int64) * 2
        m = msa.Memory(off, 2, 1, 64, 1, 64, torch.bfloat16, 1e4, 16)
        st = torch.from_numpy(np.ascontiguousarray(full[:, bounds[s]:bounds[s + 1]])).cuda()
        kc = min(k, nd)
        ids_s = torch.zeros(B, kc, dtype=torch.int32, device="cuda")
        sc_s = torch.zeros(B, kc, device="cuda")
        m.route(None, None, kc, st, ids_s, sc_s, msa.workspace(m.route_workspace_size(B, 0, kc)))
        c_id[s].fill_(-1)
        c_sc[s].fill_(float("-inf"))
        c_id[s, :, :kc] = ids_s
        c_sc[s, :, :kc] = sc_s
    g_ids, g_sc = msa.topk_merge(c_sc, c_id, bounds[:-1], k)
    want_ids, want_sc = oracle.topk(full.astype(np.float64), k)
    assert np.array_equal(g_ids.cpu().numpy(), want_ids)
    assert np.array_equal(g_sc.cpu().numpy().astype(np.float64), want_sc)


@pytest.mark.gpu
def test_merge_rejects_bad_arguments_before_any_launch():
    from top_document_sparse_b200 import msa
    c_sc = torch.zeros(2, 3, 4, device="cuda")
    c_id = torch.zeros(2, 3, 4, dtype=torch.int32, device="cuda")
    for bases, k in (([0, 5], 9), ([5, 0], 4), ([0, -1], 4), ([0, 5], 0)):
        with pytest.raises(msa.MsaError) as e:
            msa.topk_merge(c_sc, c_id, bases, k)
        assert e.value.status == 1
