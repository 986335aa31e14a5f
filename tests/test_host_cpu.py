"""Host-side checks that need no GPU: the C-ABI library builds, loads and exports
every symbol include/kalm.h declares; without a device every entry point
refuses with KALM_ERR_NO_DEVICE (no CPU fallback); document sharding and the
sharded scoring API over two gloo ranks reproduce the single-process scores in input
order, and a failure on one rank raises on every rank."""
import dataclasses
import os
import re
import socket

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(kalm_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    __graft_entry__.build()
    import encoder_decoder_document_b200 as k
    return k.load()


def test_library_exports_every_declared_symbol(lib):
    names = _declared_symbols()
    assert len(names) >= 12
    import encoder_decoder_document_b200._abi as abi
    for n in names:
        assert hasattr(lib, n), f"{n} is declared in include/ but not exported"
        assert n in abi.SIGNATURES, f"{n} has no binding signature"


def test_status_strings_and_version(lib):
    assert lib.kalm_version() == 100
    for code, name in [(0, b"KALM_OK"), (3, b"KALM_ERR_NO_DEVICE"), (5, b"KALM_ERR_TIMEOUT")]:
        assert lib.kalm_status_string(code) == name


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_no_device_is_an_explicit_error(lib):
    import encoder_decoder_document_b200 as k
    assert lib.kalm_device_check() == 3
    assert lib.kalm_linear(None, 0, None, 0, None, 0, None, 0, 0, 32, 8, None) == 3
    assert lib.kalm_chunk_pool(None, 0, None, None, 0, 8, 4, None, 0, None, 0, None) == 3
    assert lib.kalm_linear_chain(None, 0, None, 0, None, 0, None, 0, None, 0, 512, 640, 1024, 1536, None, 0,
                                 None) == 3
    # host-side size helpers need no device
    assert lib.kalm_linear_chain_sync_len(12800) == 100 and lib.kalm_linear_chain_sync_len(-1) == -1
    with pytest.raises(k.KalmError) as e:
        k.kalm_device_check()
    assert e.value.name == "KALM_ERR_NO_DEVICE"


def test_shard_documents_balanced_and_complete():
    from encoder_decoder_document_b200.sharding import shard_documents
    rng = np.random.default_rng(0)
    lens = rng.integers(1, 1025, 100)
    for world in (1, 2, 3, 8):
        shards = shard_documents(lens, world)
        allidx = np.sort(np.concatenate(shards))
        np.testing.assert_array_equal(allidx, np.arange(100))
        loads = [float((512 + lens[s]).sum()) for s in shards]
        assert max(loads) - min(loads) <= 512 + 1024  # LPT bound: one document's cost
    assert [len(s) for s in shard_documents([5], 4)] == [1, 0, 0, 0]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _oracle_rows(q):
    """score_fn for the sharded API on the CPU: the oracle's (yes, no, margin, score)
    rows of the documents it is given, as a query of their own."""
    import oracle

    def fn(x0, enc, doc_len):
        lens = np.asarray(doc_len, dtype=np.int32)
        sub = dataclasses.replace(q, x0=x0, enc=enc, doc_len=lens,
                                  tok_off=np.concatenate([[0], np.cumsum(lens, dtype=np.int64)]))
        return np.stack(oracle.forward_query(sub), 1)
    return fn


def _rank_main(rank, world, port, out, fail_rank):
    import datetime
    import torch.distributed as dist
    import synthetic
    from encoder_decoder_document_b200.sharding import sharded_rerank, sharded_scores
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    q = synthetic.make_query("tiny", hidden=64, n_docs=5)
    fn = _oracle_rows(q)
    if rank == fail_rank:
        def fn(x0, enc, doc_len):  # noqa: F811 - this rank's scoring fails on the host
            raise RuntimeError("planted failure")
    try:
        res = sharded_scores(fn, q.x0, q.enc, q.doc_len)
        ranked = sharded_rerank(fn, q.x0, q.enc, q.doc_len, top_n=3)
        out.put((rank, "ok", res, ranked))
    except RuntimeError as e:
        out.put((rank, "raised", str(e), None))
    dist.barrier()
    dist.destroy_process_group()


def _run_ranks(world, fail_rank=-1):
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out, fail_rank)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((out.get(timeout=240) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    return got


def test_two_rank_document_sharding_gloo():
    """The sharded scoring API over two gloo ranks: each rank scores its share of the
    documents, one host gather puts the rows back in input order, and every rank gets
    the whole result, equal to scoring all documents in one process."""
    import oracle
    import synthetic
    from encoder_decoder_document_b200.scorer import rank
    got = _run_ranks(2)
    q = synthetic.make_query("tiny", hidden=64, n_docs=5)
    want = np.stack(oracle.forward_query(q), 1)
    for r, status, res, ranked in got:
        assert status == "ok", res
        np.testing.assert_array_equal(res, want)
        assert ranked == rank(want[:, 2], want[:, 3], 3)


def test_sharded_scoring_failure_on_one_rank_raises_on_every_rank():
    """A rank whose scoring fails still takes part in the gather; then every rank
    raises, naming the failed rank, and no rank is left waiting in a collective."""
    got = _run_ranks(2, fail_rank=1)
    for r, status, msg, _ in got:
        assert status == "raised"
        assert "rank 1" in msg and "planted failure" in msg


def test_sharded_scores_single_process_and_slicing():
    """Without a process group the sharded call is the plain call; slice_documents
    takes documents' rows out of a packed batch."""
    import oracle
    import synthetic
    from encoder_decoder_document_b200.sharding import slice_documents, sharded_scores
    q = synthetic.make_query("tiny", hidden=64, n_docs=4)
    res = sharded_scores(_oracle_rows(q), q.x0, q.enc, q.doc_len)
    np.testing.assert_array_equal(res, np.stack(oracle.forward_query(q), 1))
    enc = np.arange(10 * 2).reshape(10, 2)
    rows, lens = slice_documents(enc, [3, 0, 5, 2], [2, 0, 1])
    np.testing.assert_array_equal(rows, np.concatenate([enc[3:8], enc[0:3]]))
    np.testing.assert_array_equal(lens, [5, 3, 0])
    rows, lens = slice_documents(enc, [3, 0, 5, 2], [])
    assert rows.shape == (0, 2) and lens.shape == (0,)
    # a query without documents: an empty (0, 4) result and an empty ranking
    from encoder_decoder_document_b200.sharding import sharded_rerank
    none = sharded_scores(_oracle_rows(q), q.x0, q.enc[:0], np.zeros(0, np.int32))
    assert none.shape == (0, 4)
    assert sharded_rerank(_oracle_rows(q), q.x0, q.enc[:0], np.zeros(0, np.int32)) == []


def _bench(args, env_extra=None):
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, **(env_extra or {}))
    res = subprocess.run([sys.executable, os.path.join(root, "bench.py"), *args], capture_output=True, text=True,
                         cwd=root, env=env, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    return [json.loads(l) for l in lines]


def test_bench_reference_arm_contract():
    """`bench.py --impl reference` times the oracle on the host cores and prints one
    JSON line with the contract's keys; ranks other than 0 print nothing."""
    (line,) = _bench(["--impl", "reference", "--config", "tiny", "--steps", "2", "--warmup", "1"])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["steps"] == 2 and line["warmup"] == 1
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert "workload" in line["config"]
    assert _bench(["--impl", "reference", "--config", "tiny", "--steps", "1", "--warmup", "0"],
                  {"RANK": "1", "WORLD_SIZE": "2"}) == []


def test_bench_accounting_with_chained_projections():
    """The bench's per-kernel work with the projections chained only regroups the work
    of the unchained stack: the same total, and the chained launches plus the first
    layer's Q|K|V and the last layer's output projection carry the unchained
    projections' FLOPs (Nano and a one-layer stack, where nothing chains)."""
    import importlib.util
    import synthetic
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    for name in ("nano", "tiny"):
        q = synthetic.make_query(name, with_weights=False)
        a, b = bench.workload(q, chain=False), bench.workload(q, chain=True)
        assert a["total_flops"] == b["total_flops"]
        assert b.get("o_proj_qkv", 0) + b["qkv_proj"] + b["o_proj"] == a["qkv_proj"] + a["o_proj"]
        assert ("o_proj_qkv" in b) == (q.layers > 1)
