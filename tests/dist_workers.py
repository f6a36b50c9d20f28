"""Process bodies for the two-rank gloo tests (spawned; not collected)."""
import datetime
import os
import sys

import numpy as np
import torch
import torch.distributed as dist


def _init(rank, world, port, timeout_s=20.0):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=timeout_s))


def imatrix_shards(rank, world, port, root, out_dir):
    sys.path.insert(0, root)
    import oracle
    import synth
    from group_scale_search_b200.dist import allreduce_imatrix, max_over_ranks, shard_range
    _init(rank, world, port)
    X = synth.make("c1", "cpu", scale=0.0625).sites["x"].X[0].float().numpy()   # same on every rank
    T = X.shape[0]
    t0, t1 = shard_range(T, rank, world)
    local = oracle.imatrix(X[t0:t1]) * (t1 - t0)          # this rank's raw sums of x^2
    m = allreduce_imatrix(torch.from_numpy(local.astype(np.float32)), T)
    slowest = max_over_ranks(float(rank + 1))
    np.save(os.path.join(out_dir, f"m{rank}.npy"), m.numpy())
    np.save(os.path.join(out_dir, f"t{rank}.npy"), np.array([slowest]))
    dist.barrier()
    dist.destroy_process_group()


def proxy_row_shards(rank, world, port, root, out_dir):
    """Each rank takes half of the rows of every matrix and reduces its
    (num, den); the all-reduced sums are the whole matrices'."""
    sys.path.insert(0, root)
    import oracle
    from group_scale_search_b200.dist import allreduce_proxy, shard_range
    _init(rank, world, port)
    rng = np.random.default_rng(4)                      # same data on every rank
    E, O, I = 3, 37, 200
    W = (rng.standard_t(4, size=(E, O, I)) * 0.02).astype(np.float32)
    What = (W + rng.normal(0, 1e-3, size=W.shape)).astype(np.float32)
    m = rng.lognormal(0, 1, size=(E, I)).astype(np.float32)
    o0, o1 = shard_range(O, rank, world)
    nums, dens = [], []
    for e in range(E):
        n, d = oracle.proxy_error(W[e, o0:o1], What[e, o0:o1], m[e])
        nums.append(n)
        dens.append(d)
    num, den = allreduce_proxy(torch.tensor(nums, dtype=torch.float64), torch.tensor(dens, dtype=torch.float64))
    np.save(os.path.join(out_dir, f"p{rank}.npy"), np.stack([num.numpy(), den.numpy()]))
    dist.barrier()
    dist.destroy_process_group()


def hessian_gptq_shards(rank, world, port, root, out_dir):
    """Token-sharded calibration: each rank forms X_r^T X_r of its tokens,
    the all-reduce gives every rank the whole H; each rank then sweeps its
    own rows of W (GPTQ with the factor of the damped H^-1) with no exchange,
    and the token-sharded full-Hessian proxy error of the result goes through
    allreduce_proxy.  The oracle stands in for the GPU calls (host logic)."""
    sys.path.insert(0, root)
    import oracle
    from group_scale_search_b200.dist import allreduce_hessian, allreduce_proxy, shard_range
    _init(rank, world, port)
    rng = np.random.default_rng(8)                      # same data on every rank
    T, O, I = 96, 21, 160
    X = rng.standard_normal((T, I)).astype(np.float32)
    W = (rng.standard_t(4, size=(O, I)) * 0.02).astype(np.float32)
    t0, t1 = shard_range(T, rank, world)
    H = allreduce_hessian(torch.from_numpy(oracle.hessian(X[t0:t1]))).numpy()
    Hd = H + 0.01 * np.mean(np.diag(H)) * np.eye(I)
    U = np.ascontiguousarray(np.linalg.cholesky(np.linalg.inv(Hd)).T.astype(np.float32))
    s, z = [a[0] for a in oracle.search_asym_int4(W[None], np.diag(H).astype(np.float32) / T)[:2]]
    o0, o1 = shard_range(O, rank, world)
    codes, _ = oracle.gptq_sweep(W[o0:o1], 4, s[o0:o1], z[o0:o1], U)
    # every rank needs every (row shard, token shard) pair: gather the row shards' codes first
    rows = [shard_range(O, r, world) for r in range(world)]
    pad = max(b - a for a, b in rows)                    # gloo gathers equal sizes: pad, then trim
    mine = torch.zeros((pad, I), dtype=torch.int8)
    mine[: o1 - o0] = torch.from_numpy(codes)
    allc = [torch.zeros((pad, I), dtype=torch.int8) for _ in range(world)]
    dist.all_gather(allc, mine)
    allc = [c[: b - a] for c, (a, b) in zip(allc, rows)]
    Wq = oracle.dequant_int4(torch.cat(allc).numpy().astype(np.uint8), s, z)
    n, d = oracle.proxy_error_full(W, Wq, oracle.hessian(X[t0:t1]))            # all rows x this rank's tokens
    num, den = allreduce_proxy(torch.tensor([n], dtype=torch.float64), torch.tensor([d], dtype=torch.float64))
    np.save(os.path.join(out_dir, f"h{rank}.npy"), H)
    np.save(os.path.join(out_dir, f"c{rank}.npy"), torch.cat(allc).numpy())
    np.save(os.path.join(out_dir, f"q{rank}.npy"), np.array([num.item(), den.item()]))
    dist.barrier()
    dist.destroy_process_group()


def peer_dies(rank, world, port, out_dir):
    """Rank 1 leaves before the collective; rank 0 must get an error, not hang."""
    _init(rank, world, port, timeout_s=8.0)
    if rank == 1:
        os._exit(0)
    t = torch.ones(4)
    try:
        dist.all_reduce(t)
        status = "completed"
    except Exception as e:   # noqa: BLE001 -- any error is the expected outcome
        status = "error: " + type(e).__name__
    with open(os.path.join(out_dir, "status.txt"), "w") as f:
        f.write(status)
    os._exit(0)


class _HostStandIn:
    """A host stand-in for the library's four step calls, used only to check
    bench.py's sharding and exchanges on CPU: deterministic per-group and
    per-column arithmetic in torch (not the method), so that a sharded run
    can be compared with a one-process run of the same inputs."""
    FORMATS = {"int3_g64_sym": 5, "int4_g128_asym": 4, "nvfp4_g16": 16}
    GROUP = {5: 64, 4: 128, 16: 16}

    class Result:
        def __init__(self, scales):
            self.scales, self.zeros, self.global_scale, self.packed = scales, None, None, scales
            self.cand_idx = self.loss = None

    def imatrix_workspace_bytes(self, X):
        return 16

    def proxy_workspace_bytes(self, W, fmt):
        return 16

    def tq_imatrix(self, X, m, alpha, workspace=None):
        m.copy_((X.double().square().sum(dim=1) * alpha).float())
        return m

    def search_result_empty(self, W, fmt, want_idx=True, want_loss=True):
        E, O, I = W.shape
        G = -(-I // self.GROUP[fmt])
        return self.Result(torch.empty((E, O, G), dtype=torch.float32))

    def tq_search_groups(self, W, m, fmt, want_idx=True, want_loss=True, out=None):
        E, O, I = W.shape
        g = self.GROUP[fmt]
        G = -(-I // g)
        pad = torch.nn.functional.pad(W.float().abs(), (0, G * g - I))
        s = pad.reshape(E, O, G, g).amax(dim=3)
        if out is None:
            return self.Result(s)
        out.scales.copy_(s)
        return out

    def tq_dequant(self, packed, fmt, scales, zeros, gs, E, O, I, out):
        g = self.GROUP[fmt]
        out.copy_(scales.repeat_interleave(g, dim=2)[:, :, :I].to(out.dtype))
        return out

    def proxy_batch_workspace_bytes(self, Ws, fmt):
        return 16

    def tq_dequant_batch(self, packed, fmt, scales, zeros, gs, shapes, out):
        for i, (E, O, I) in enumerate(shapes):
            self.tq_dequant(packed[i], fmt, scales[i], None, None, E, O, I, out=out[i])
        return out

    def tq_proxy_error_batch(self, Ws, packed, fmt, scales, zeros, gs, ms, out, workspace=None):
        for i, W in enumerate(Ws):
            self.tq_proxy_error(W, packed[i], fmt, scales[i], None, None, ms[i], out=out[i])
        return out

    def tq_proxy_error(self, W, packed, fmt, scales, zeros, gs, m, out, workspace=None):
        mm = m if m.dim() == 2 else m.unsqueeze(0)
        w = W.double()
        out[0].copy_((w.square() * mm.double().unsqueeze(1)).sum(dim=(1, 2)))
        out[1].copy_((w.abs() * mm.double().unsqueeze(1)).sum(dim=(1, 2)))
        return out


def bench_sharded_step(rank, world, port, root, out_dir, config):
    """bench.py's strong-scaling split of `config` (scale 0.05) over gloo ranks:
    this rank's part, one step with the host stand-in, results saved for the
    parent to compare with a one-process run."""
    sys.path.insert(0, root)
    import bench
    import synth
    _init(rank, world, port)
    wl = synth.make(config, "cpu", seed=0, scale=0.05)
    part, shard = bench.shard_workload(wl, world, rank)
    step = bench.Step(_HostStandIn(), part, bench.make_sets(part, 1), shard)
    step(0)
    out = {"m": {k: v.numpy() for k, v in step.m.items()},
           "scales": [r.scales.numpy() for r in step.res],
           "px": [np.stack([a.numpy(), b.numpy()]) for a, b in step.px],
           "pieces": shard.pieces}
    np.save(os.path.join(out_dir, f"s{rank}.npy"), np.array([out], dtype=object), allow_pickle=True)
    dist.barrier()
    dist.destroy_process_group()
