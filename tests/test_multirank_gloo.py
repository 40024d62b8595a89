"""The multi-process (one rank per GPU) host logic, run as world_size-2 `gloo`
process groups on the CPU: the max-over-ranks timing reduction, the
rank-specific seeds of a weak-scaling run, and head sharding.  The op has no
collective on its data path: every (b, h) pair is independent, so a head
split computed rank by rank (here with the float64 oracle) and gathered must
equal the whole computation."""

import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

from frame_wise_delta_vda_b200 import inputs as gen  # noqa: E402
from frame_wise_delta_vda_b200 import ranks  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, fn, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        q.put((rank, fn(rank, world)))
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, e))
    finally:
        dist.destroy_process_group()


def _spawn(fn, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, fn, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, v in res.items():
        if isinstance(v, Exception):
            raise v
    return res


def _max_fn(rank, world):
    return ranks.max_over_ranks(1.5 + rank, dist)


def test_max_over_ranks_gloo():
    res = _spawn(_max_fn)
    assert res == {0: 2.5, 1: 2.5}


def test_max_over_ranks_single_process():
    assert ranks.max_over_ranks(3.25, None) == 3.25


def test_rank_seeds_are_distinct_and_stable():
    seeds = [ranks.rank_seed(3, r) for r in range(8)]
    assert len(set(seeds)) == 8 and seeds[0] == 3
    assert seeds == [ranks.rank_seed(3, r) for r in range(8)]


@pytest.mark.parametrize("B,H,world", [(1, 48, 8), (2, 48, 3), (1, 5, 4), (1, 2, 2), (3, 1, 2)])
def test_head_shard_partitions_every_head_once(B, H, world):
    owned = [p for r in range(world) for p in ranks.head_shard(B, H, r, world)]
    assert owned == [(b, h) for b in range(B) for h in range(H)]
    sizes = [len(ranks.head_shard(B, H, r, world)) for r in range(world)]
    assert max(sizes) - min(sizes) <= 1


def _shard_fn(rank, world):
    import oracle as ref
    wl = gen.custom("shard", H=3, T=6, U=5, d=4, chunk=2, window_chunks=0, dtype="f32", seed=7)
    mine = ranks.head_shard(wl.B, wl.H, rank, world)
    x = gen.make_inputs(wl, heads=mine)
    y = ref.vda_forward(x["q"][None], x["k"][None], x["v"][None], x["beta"][None], x["gate"][None],
                        x["rms_weight"], None, None, wl.chunk, wl.window_chunks,
                        heads=[(0, i) for i in range(len(mine))])
    # gather the variable-size shards: pad to the largest shard, then trim
    n_max = -(-wl.B * wl.H // world)
    buf = np.zeros((n_max,) + y.shape[1:])
    buf[:len(mine)] = y
    parts = [torch.zeros(buf.shape, dtype=torch.float64) for _ in range(world)]
    dist.all_gather(parts, torch.from_numpy(buf))
    sizes = [len(ranks.head_shard(wl.B, wl.H, r, world)) for r in range(world)]
    return np.concatenate([p.numpy()[:n] for p, n in zip(parts, sizes)])


def test_head_sharded_run_equals_whole_run_gloo():
    import oracle as ref
    res = _spawn(_shard_fn)
    wl = gen.custom("shard", H=3, T=6, U=5, d=4, chunk=2, window_chunks=0, dtype="f32", seed=7)
    x = gen.make_inputs(wl)
    y = ref.vda_forward(x["q"], x["k"], x["v"], x["beta"], x["gate"], x["rms_weight"], None, None,
                        wl.chunk, wl.window_chunks).reshape((wl.B * wl.H,) + (wl.T, wl.U, wl.d))
    for r in range(2):
        np.testing.assert_array_equal(res[r], y)


# --- the Ulysses layout: sequence shards <-> head shards around the op ---------
UWL = dict(B=1, H=4, T=6, U=10, d=16, chunk=2, window_chunks=1, dtype="f32", seed=9, alpha_mean=2.0)


def _ulysses_round_trip_fn(rank, world):
    from frame_wise_delta_vda_b200 import ulysses
    B, H, T, U, d = 2, 4, 3, 4, 8
    g = torch.Generator().manual_seed(5)
    full = torch.randn(B, H, T, U, d, generator=g).to(torch.bfloat16)
    seq = ulysses.token_shard(full, rank, world, T, U)
    heads = ulysses.seq_to_heads(seq)
    Hp = H // world
    want = full[:, rank * Hp:(rank + 1) * Hp].reshape(B, Hp, T * U, d)
    assert torch.equal(heads.view(torch.int16), want.view(torch.int16))
    back = ulysses.heads_to_seq(heads)
    assert torch.equal(back.view(torch.int16), seq.view(torch.int16))
    return True


def test_ulysses_exchange_round_trip_gloo():
    assert _spawn(_ulysses_round_trip_fn) == {0: True, 1: True}


def _oracle_forward(q, k, v, beta, gate, w, S0f, S0r, chunk, window_chunks, alpha=None):
    """The float64 oracle on a head shard (torch tensors in, torch out)."""
    import oracle as ref
    B, Hs = q.shape[:2]
    out = np.zeros(tuple(q.shape[:-1]) + (v.shape[-1],))
    for b in range(B):
        for h in range(Hs):
            s0f = None if S0f is None else S0f[b, h].double().numpy()
            s0r = None if S0r is None else S0r[b, h].double().numpy()
            a = None if alpha is None else alpha[b, h].double().numpy()
            out[b, h] = ref.vda_forward_head(q[b, h].double().numpy(), k[b, h].double().numpy(),
                                             v[b, h].double().numpy(), beta[b, h].double().numpy(),
                                             gate[b, h].double().numpy(), w.double().numpy(), s0f, s0r,
                                             chunk, window_chunks, alpha=a)
    return torch.from_numpy(out)


def _ulysses_forward_fn(rank, world):
    from frame_wise_delta_vda_b200 import ulysses
    wl = gen.custom("ulysses", **UWL)
    x = {k: torch.from_numpy(np.ascontiguousarray(v)) for k, v in gen.make_inputs(wl).items()}
    rng = np.random.default_rng(11)
    S0 = torch.from_numpy(0.3 * rng.standard_normal((wl.B, wl.H, wl.d, wl.d)))
    Hp = wl.H // world
    sh = lambda t: ulysses.token_shard(t, rank, world, wl.T, wl.U)
    out = ulysses.vda_forward_ulysses(sh(x["q"]), sh(x["k"]), sh(x["v"]), sh(x["beta"]), sh(x["gate"]),
                                      x["rms_weight"], S0[:, rank * Hp:(rank + 1) * Hp],
                                      S0[:, rank * Hp:(rank + 1) * Hp], wl.T, wl.U, wl.chunk, wl.window_chunks,
                                      alpha=x["alpha"][:, rank * Hp:(rank + 1) * Hp], forward=_oracle_forward)
    return out.numpy()   # [B, H, S/P, d]: every head, this rank's tokens


def test_ulysses_sharded_forward_equals_unsharded_oracle_gloo():
    """Sequence shards exchanged into head shards, the oracle per rank, the
    outputs exchanged back: bit for bit the unsharded oracle (the exchange
    moves bits; each head's arithmetic is the same)."""
    import oracle as ref
    res = _spawn(_ulysses_forward_fn)
    wl = gen.custom("ulysses", **UWL)
    x = gen.make_inputs(wl)
    rng = np.random.default_rng(11)
    S0 = 0.3 * rng.standard_normal((wl.B, wl.H, wl.d, wl.d))
    y = np.zeros((wl.B, wl.H, wl.T, wl.U, wl.d))
    for h in range(wl.H):
        y[0, h] = ref.vda_forward_head(gen.as_f64(x["q"][0, h]), gen.as_f64(x["k"][0, h]), gen.as_f64(x["v"][0, h]),
                                       x["beta"][0, h], gen.as_f64(x["gate"][0, h]), x["rms_weight"],
                                       S0[0, h], S0[0, h], wl.chunk, wl.window_chunks,
                                       alpha=gen.as_f64(x["alpha"][0, h]))
    y = y.reshape(wl.B, wl.H, wl.T * wl.U, wl.d)
    n = wl.T * wl.U // 2
    for r in range(2):
        np.testing.assert_array_equal(res[r], y[:, :, r * n:(r + 1) * n])
