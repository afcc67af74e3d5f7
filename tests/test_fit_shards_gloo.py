"""The closed-form fit across ranks (bench.py --fit under torchrun), on CPU: each of two gloo
ranks adds the normal-equation and scale sums of its shard of the calibration prompts, one
all-reduce joins them, and the result equals the sums of all prompts taken in one process.
The sums here are the oracle's, over synthetic codes; the GPU path adds the same sums with
its own kernels and joins them with the same call."""
import os
import socket
import sys

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
N_PROMPTS = 5  # uneven over two ranks


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _prompt(i):
    """Prompt i: 132 + 3 + i tokens, token ids, codes and centres (seeded)."""
    import oracle as O

    rng = np.random.default_rng(100 + i)
    n = 3 + i
    tok = rng.integers(0, 8, size=132 + n)
    q = rng.integers(-300, 300, size=(n, O.N_COEF))
    c = rng.integers(-5, 6, size=(n, O.N_COEF))
    return tok, dict(qe=q[0::2], qo=q[1::2], ce=c[0::2], co=c[1::2])


def _sums(ids):
    """Flat tensors of the even-model sums (G_e, C_e, row counts) and the scale sums."""
    import oracle as O

    rng = np.random.default_rng(7)
    emb = rng.standard_normal((8, O.N_COEF)).astype(np.float32).view(np.uint32) >> 16
    emb = emb.astype(np.uint16)
    toks, codes = zip(*[_prompt(i) for i in ids]) if ids else ((), ())
    offs = np.concatenate([[0], np.cumsum([len(t) for t in toks])]).astype(np.int64)
    tok = np.concatenate(toks) if toks else np.zeros(0, np.int64)
    st = O.fit_statistics_from_codes(list(codes), tok, offs, emb)
    b = np.ones(O.N_COEF, np.float32)
    d = np.ones(O.N_COEF, np.float32)
    b[3] = 0.01  # one dropped component
    total, rows = O.fit_scales_from_codes(list(codes), b, d)
    f = torch.from_numpy(np.concatenate([st["g_e"].ravel(), st["c_e"].ravel(), [st["n_e"], st["n_o"]]]))
    i = torch.from_numpy(np.concatenate([total, [rows]]).astype(np.int64))
    return f, i


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = bench.fit_shard(range(N_PROMPTS), rank, world)
        f, i = _sums(mine)
        bench.fit_allreduce(f, dist)
        bench.fit_allreduce(i, dist)
        np.save(os.path.join(out_dir, f"f{rank}.npy"), f.numpy())
        np.save(os.path.join(out_dir, f"i{rank}.npy"), i.numpy())
        np.save(os.path.join(out_dir, f"ids{rank}.npy"), np.array(mine))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_sharded_sums_equal_the_whole_batch(tmp_path):
    sys.path.insert(0, ROOT)
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    ids = [list(np.load(tmp_path / f"ids{r}.npy")) for r in range(world)]
    assert sorted(ids[0] + ids[1]) == list(range(N_PROMPTS)) and not set(ids[0]) & set(ids[1])
    f_all, i_all = _sums(list(range(N_PROMPTS)))
    for r in range(world):
        f = np.load(tmp_path / f"f{r}.npy")
        i = np.load(tmp_path / f"i{r}.npy")
        assert np.array_equal(i, i_all.numpy())  # integer sums: exact
        assert np.allclose(f, f_all.numpy(), rtol=1e-12, atol=1e-9)  # fp64 sums in another order
        assert f[-2] == f_all[-2] and f[-1] == f_all[-1]  # row counts


def test_single_process_sums_are_the_total():
    sys.path.insert(0, ROOT)
    import bench

    t = torch.arange(4, dtype=torch.float64)
    assert bench.fit_allreduce(t) is t and torch.equal(t, torch.arange(4, dtype=torch.float64))
    assert bench.fit_shard(range(5), 1, 2) == [1, 3]
