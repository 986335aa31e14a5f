"""Document-sharded reranking through the product path: two ranks (one process each,
gloo for the host gather), each with its own scorer, score their shares of one query's
documents and gather the rows back in input order.  Both ranks share the one GPU of the
test box; their kernels never wait on each other (the only exchange is the host gather).
"""
import datetime

import numpy as np
import pytest

import oracle
import synthetic

pytestmark = pytest.mark.gpu

SCORE_TOL = 1e-3   # scores end to end at two layers
RANK_GAP = 1e-2    # pairs the oracle separates by more than this keep their order


def _query():
    return synthetic.make_query("nano", n_docs=7, layers=2)


def _rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist
    from encoder_decoder_document_b200.scorer import DeviceWeights, FBNLScorer
    from encoder_decoder_document_b200.sharding import shard_documents, sharded_scores
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    # every rank takes the same collective steps and always reports, also when it fails
    try:
        q = _query()
        sc = FBNLScorer(DeviceWeights.from_bits(q.weights), q.n_q, q.n_kv)
        fn = sc.score_rows
    except Exception as e:
        q, fn = _query(), None
        err = f"{type(e).__name__}: {e}"

    def rows(x0, enc, doc_len):
        if fn is None:
            raise RuntimeError(err)
        return fn(x0, enc, doc_len)
    try:
        res = sharded_scores(rows, q.x0, q.enc, q.doc_len)
        ranked = sc.rerank_sharded(q.x0, q.enc, q.doc_len, top_n=4)
        out.put((rank, res, ranked, shard_documents(q.doc_len, world)[rank]))
    except Exception as e:
        out.put((rank, None, f"{type(e).__name__}: {e}", None))
    dist.barrier()
    dist.destroy_process_group()


def _free_port():
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_rerank_sharded_two_ranks_matches_one_process_and_oracle():
    import multiprocessing as mp
    import torch
    from encoder_decoder_document_b200.scorer import DeviceWeights, FBNLScorer, rank
    q = _query()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted((out.get(timeout=600) for _ in range(2)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r, res, msg, _ in got:
        assert res is not None, f"rank {r}: {msg}"
    # each rank scored a non-empty share, and the shares cover every document once
    shares = [g[3] for g in got]
    assert all(len(s) for s in shares)
    np.testing.assert_array_equal(np.sort(np.concatenate(shares)), np.arange(q.n_docs))
    # one process over all documents: a document's rows do not depend on its batch
    sc = FBNLScorer(DeviceWeights.from_bits(q.weights), q.n_q, q.n_kv)
    whole = sc.score_rows(q.x0, q.enc, q.doc_len)
    torch.cuda.synchronize()
    y, n, m, s = oracle.forward_query(q)
    for r, res, ranked, _ in got:
        np.testing.assert_array_equal(res, whole)
        assert ranked == rank(whole[:, 2], whole[:, 3], 4)
        assert np.abs(res[:, 3] - s).max() <= SCORE_TOL
        for i in range(q.n_docs):
            for j in range(q.n_docs):
                if s[i] - s[j] > RANK_GAP:
                    assert res[i, 3] > res[j, 3]


def test_rerank_sharded_without_process_group_is_rerank():
    from encoder_decoder_document_b200.scorer import DeviceWeights, FBNLScorer
    q = _query()
    sc = FBNLScorer(DeviceWeights.from_bits(q.weights), q.n_q, q.n_kv)
    assert sc.rerank_sharded(q.x0, q.enc, q.doc_len) == sc.rerank(q.x0, q.enc, q.doc_len)
    empty = sc.score_rows(q.x0, q.enc[:0], np.zeros(0, np.int32))
    assert empty.shape == (0, 4)
