"""Multi-process (N > 1) host path on CPU with gloo ranks: work sharding,
token-sharded imatrix all-reduce, row-sharded proxy-error all-reduce,
token-sharded Hessian then row-sharded GPTQ sweep and full-Hessian proxy error,
max-over-ranks timing, and a rank that dies before a collective (the
survivor must fail fast, not hang)."""
import multiprocessing as mp
import os
import socket
import time

import numpy as np

import dist_workers
from group_scale_search_b200.dist import shard_range, shard_units

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run(target, args, world=2, timeout=120):
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=target, args=(r, world) + args) for r in range(world)]
    for p in procs:
        p.start()
    deadline = time.time() + timeout
    for p in procs:
        p.join(max(1.0, deadline - time.time()))
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive, "a rank hung"
    return [p.exitcode for p in procs]


def test_shard_range_covers_everything_once():
    for n in (0, 1, 7, 4096, 65536):
        for world in (1, 2, 3, 8):
            spans = [shard_range(n, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1


def test_shard_units_balances_the_27b_layer():
    # the 7 linears of the 27B-dense layer, cost = weights
    costs = [5120 * 5120, 1024 * 5120, 1024 * 5120, 5120 * 5120, 17408 * 5120, 17408 * 5120, 5120 * 17408]
    for world in (1, 2, 4, 8):
        plan = shard_units(costs, world)
        assert sorted(i for p in plan for i in p) == list(range(7))
        loads = [sum(costs[i] for i in p) for p in plan]
        assert max(loads) <= max(costs) + sum(costs) / world


def test_token_sharded_imatrix_allreduce(tmp_path):
    import oracle
    import synth
    codes = _run(dist_workers.imatrix_shards, (_port(), ROOT, str(tmp_path)))
    assert codes == [0, 0]
    X = synth.make("c1", "cpu", scale=0.0625).sites["x"].X[0].float().numpy()
    ref = oracle.imatrix(X)
    for r in range(2):
        m = np.load(tmp_path / f"m{r}.npy")
        assert np.max(np.abs(m - ref) / ref) <= 1e-6
        assert np.load(tmp_path / f"t{r}.npy")[0] == 2.0      # max over ranks of (rank + 1)


def test_row_sharded_proxy_allreduce(tmp_path):
    import oracle
    codes = _run(dist_workers.proxy_row_shards, (_port(), ROOT, str(tmp_path)))
    assert codes == [0, 0]
    rng = np.random.default_rng(4)
    E, O, I = 3, 37, 200
    W = (rng.standard_t(4, size=(E, O, I)) * 0.02).astype(np.float32)
    What = (W + rng.normal(0, 1e-3, size=W.shape)).astype(np.float32)
    m = rng.lognormal(0, 1, size=(E, I)).astype(np.float32)
    ref = np.array([oracle.proxy_error(W[e], What[e], m[e]) for e in range(E)]).T
    for r in range(2):
        got = np.load(tmp_path / f"p{r}.npy")
        assert np.max(np.abs(got - ref) / ref) <= 1e-12      # fp64 sums of two halves


def test_token_sharded_hessian_then_row_sharded_gptq(tmp_path):
    """The full-Hessian path on 2 ranks: the all-reduced H equals X^T X of all
    tokens, the row-sharded sweeps gathered equal the one-process sweep bit
    for bit, and the token-sharded tr(E H E^T), tr(W H W^T) equal the whole."""
    import oracle
    codes = _run(dist_workers.hessian_gptq_shards, (_port(), ROOT, str(tmp_path)))
    assert codes == [0, 0]
    rng = np.random.default_rng(8)
    T, O, I = 96, 21, 160
    X = rng.standard_normal((T, I)).astype(np.float32)
    W = (rng.standard_t(4, size=(O, I)) * 0.02).astype(np.float32)
    H = oracle.hessian(X)
    Hd = H + 0.01 * np.mean(np.diag(H)) * np.eye(I)
    U = np.ascontiguousarray(np.linalg.cholesky(np.linalg.inv(Hd)).T.astype(np.float32))
    s, z = [a[0] for a in oracle.search_asym_int4(W[None], np.diag(H).astype(np.float32) / T)[:2]]
    ref_codes, _ = oracle.gptq_sweep(W, 4, s, z, U)
    ref = oracle.proxy_error_full(W, oracle.dequant_int4(ref_codes.astype(np.uint8), s, z), H)
    for r in range(2):
        assert np.allclose(np.load(tmp_path / f"h{r}.npy"), H, rtol=1e-13, atol=1e-10)
        assert np.array_equal(np.load(tmp_path / f"c{r}.npy"), ref_codes)
        assert np.allclose(np.load(tmp_path / f"q{r}.npy"), ref, rtol=1e-12)


def test_surviving_rank_fails_fast_when_a_peer_dies(tmp_path):
    codes = _run(dist_workers.peer_dies, (_port(), str(tmp_path)), timeout=60)
    assert codes == [0, 0]
    status = (tmp_path / "status.txt").read_text()
    assert status.startswith("error"), status
