"""The multi-GPU partitions of compressed_long_context_hca_b200.parallel on CPU ranks.

The partition and exchange logic under test is the product's (ranges, all-gathers, halo
assembly, the order of collectives); the compute steps run on an oracle-backed backend
(float64 NumPy), so each partitioned result can be compared element by element with the
single-rank oracle. World sizes 2 and 3 over gloo on 127.0.0.1.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from compressed_long_context_hca_b200 import parallel as P
from oracle import hca_oracle as orc


# ------------------------------------------------------------------------------ ranges
@pytest.mark.parametrize("n,world,align", [(700, 3, 16), (128, 4, 128), (5, 8, 1),
                                           (1000, 2, 128), (0, 3, 16)])
def test_split_range_tiles_the_items(n, world, align):
    rs = [P.split_range(n, world, r, align) for r in range(world)]
    assert rs[0][0] == 0 and rs[-1][1] == n
    for (a, b), (c, d) in zip(rs, rs[1:]):
        assert b == c
    for a, b in rs:
        assert a % align == 0 or a == n
    units = [-(-(b - a) // align) for a, b in rs]
    assert max(units) - min(units) <= 1


def test_seq_and_entry_ranges():
    assert [P.seq_range(10, 3, r) for r in range(3)] == [(0, 4), (4, 7), (7, 10)]
    er = [P.entry_range(8191, 8, r) for r in range(8)]
    assert all(lo % 128 == 0 for lo, _ in er)
    assert er[0][0] == 0 and er[-1][1] >= 8191
    assert all(b == c for (_, b), (c, _) in zip(er, er[1:]))


# ------------------------------------------------------------------------------ backend
class OracleBackend:
    """The compute steps of parallel.py restated by the float64 oracle."""

    def __init__(self, scale):
        self.scale = scale

    def compress(self, K, V, block):
        Kc = np.stack([orc.compress_blocks(K[b].numpy(), block) for b in range(K.shape[0])])
        Vc = np.stack([orc.compress_blocks(V[b].numpy(), block) for b in range(V.shape[0])])
        return torch.from_numpy(Kc), torch.from_numpy(Vc)

    def prefill_range(self, Q, K, V, Kc, Vc, q_pos0, kv_pos0, block, window, G=None,
                      desc=None, out=None):
        b, T, hq, D = Q.shape
        out = np.zeros((b, T, hq, V.shape[-1]))
        for bi in range(b):
            # raw tokens laid out at their absolute positions (nothing before kv_pos0)
            Kabs = np.zeros((kv_pos0 + K.shape[1],) + tuple(K.shape[2:]))
            Vabs = np.zeros((kv_pos0 + V.shape[1],) + tuple(V.shape[2:]))
            Kabs[kv_pos0:] = K[bi].numpy()
            Vabs[kv_pos0:] = V[bi].numpy()
            for t in range(T):
                o, _ = orc.attend_position(Q[bi, t].numpy(), Kc[bi].numpy(), Vc[bi].numpy(),
                                           Kabs, Vabs, q_pos0 + t, block, window, self.scale)
                out[bi, t] = o if G is None else o * G[bi, t].numpy()
        return torch.from_numpy(out)

    def decode_partial(self, q, ctx_len, cache, ring_k, ring_v, e0, e1, with_window, desc):
        block, window = desc["block"], desc["window"]
        nseq, hq, D = q.shape
        out = np.zeros((nseq, hq, 2 + D))
        for b in range(nseq):
            t = int(ctx_len[b]) - 1
            nc = orc.visible_compressed_count(t, block, window)
            hi = min(e1, nc)
            keys = [cache["k"][b][j] for j in range(e0, hi)]   # this rank's shard only
            vals = [cache["v"][b][j] for j in range(e0, hi)]
            if with_window:
                lo_w, hi_w = orc.window_bounds(t, window)
                keys += [ring_k[b, u % window, 0].numpy() for u in range(lo_w, hi_w + 1)]
                vals += [ring_v[b, u % window, 0].numpy() for u in range(lo_w, hi_w + 1)]
            keys = np.array(keys).reshape(-1, D)
            vals = np.array(vals).reshape(-1, D)
            m, l, o = orc.attend_part(q[b].numpy(), keys, vals, self.scale)
            out[b, :, 0], out[b, :, 1], out[b, :, 2:] = m, l, o
        return torch.from_numpy(out)

    def decode(self, q, ctx_len, cache, ring_k, ring_v, desc):
        parts = self.decode_partial(q, ctx_len, cache, ring_k, ring_v, 0, 1 << 30, True, desc)
        return self.merge(parts[None], desc)

    def merge(self, parts, desc):
        parts = parts.numpy()
        nseq = parts.shape[1]
        O = []
        for b in range(nseq):
            o, _ = orc.merge_parts(parts[:, b, :, 0], parts[:, b, :, 1], parts[:, b, :, 2:])
            g = desc.get("gate")
            O.append(o if g is None else o * g[b])
        return torch.from_numpy(np.stack(O))


# ------------------------------------------------------------------------------ ranks
def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


PF = dict(b=2, T=700, hq=4, D=32, block=16, window=40)
DC = dict(nseq=3, hq=4, D=32, block=16, window=40)


def _prefill_inputs():
    g = torch.Generator().manual_seed(7)
    b, T, hq, D = PF["b"], PF["T"], PF["hq"], PF["D"]
    Q = torch.randn((b, T, hq, D), generator=g, dtype=torch.float64)
    K = torch.randn((b, T, 1, D), generator=g, dtype=torch.float64)
    V = torch.randn((b, T, 1, D), generator=g, dtype=torch.float64)
    G = torch.sigmoid(torch.randn((b, T, hq, D), generator=g, dtype=torch.float64))
    return Q, K, V, G


def _decode_inputs():
    g = torch.Generator().manual_seed(9)
    n, hq, D, W, blk = DC["nseq"], DC["hq"], DC["D"], DC["window"], DC["block"]
    ctx = torch.tensor([700, 5000, 8190])
    n_ent = (int(ctx.max()) - W) // blk + 1
    q = torch.randn((n, hq, D), generator=g, dtype=torch.float64)
    ek = torch.randn((n, n_ent, D), generator=g, dtype=torch.float64)
    ev = torch.randn((n, n_ent, D), generator=g, dtype=torch.float64)
    rk = torch.randn((n, W, 1, D), generator=g, dtype=torch.float64)
    rv = torch.randn((n, W, 1, D), generator=g, dtype=torch.float64)
    G = torch.sigmoid(torch.randn((n, hq, D), generator=g, dtype=torch.float64))
    return ctx, q, ek, ev, rk, rv, G


def _rank(rank, world, port, outdir):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        scale = 1.0 / np.sqrt(PF["D"])
        be = OracleBackend(scale)
        # row-partitioned prefill: this rank holds only its rows of Q, K, V, G
        Q, K, V, G = _prefill_inputs()
        t0, t1 = P.row_range(PF["T"], world, rank, PF["block"])
        O_r = P.prefill_rows(be, None, Q[:, t0:t1], K[:, t0:t1], V[:, t0:t1], PF["T"],
                             PF["block"], PF["window"], G=G[:, t0:t1])
        # split-entries decode: this rank's cache shard holds entries [e0, e1) only
        ctx, q, ek, ev, rk, rv, Gd = _decode_inputs()
        n_vis = max(orc.visible_compressed_count(int(c) - 1, DC["block"], DC["window"])
                    for c in ctx)
        e0, e1 = P.entry_range(n_vis, world, rank)
        shard = {"k": [{j: ek[b, j].numpy() for j in range(e0, min(e1, ek.shape[1]))}
                       for b in range(DC["nseq"])],
                 "v": [{j: ev[b, j].numpy() for j in range(e0, min(e1, ev.shape[1]))}
                       for b in range(DC["nseq"])]}
        last = rank == world - 1
        desc = {"block": DC["block"], "window": DC["window"], "gate": Gd.numpy()}
        Od = P.decode_split_entries(be, None, q, ctx, shard, rk if last else None,
                                    rv if last else None, n_vis, desc)
        # results go through files: a queue's pipe would block the rank until the parent,
        # still joining, reads it
        np.savez(os.path.join(outdir, f"rank{rank}.npz"), O_r=O_r.numpy(), Od=Od.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [1, 2, 3])
def test_partitions_match_single_rank_oracle(world, tmp_path):
    mp.start_processes(_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = []
    for r in range(world):
        z = np.load(os.path.join(tmp_path, f"rank{r}.npz"))
        res.append((r, None, z["O_r"], z["Od"]))
    scale = 1.0 / np.sqrt(PF["D"])
    # prefill rows, reassembled, against the whole-sequence oracle
    Q, K, V, G = _prefill_inputs()
    O = np.concatenate([r[2] for r in res], axis=1)
    assert O.shape[1] == PF["T"]
    for b in range(PF["b"]):
        ref, _ = orc.hca_prefill(Q[b].numpy(), K[b].numpy(), V[b].numpy(), PF["block"],
                                 PF["window"], scale, gate=G[b].numpy())
        assert np.abs(O[b] - ref).max() <= 1e-12
    # decode: every rank holds the same merged output, equal to the whole-key-set oracle
    ctx, q, ek, ev, rk, rv, Gd = _decode_inputs()
    for b in range(DC["nseq"]):
        ref, _ = orc.hca_decode(q[b].numpy(), ek[b, :, None].numpy(), ev[b, :, None].numpy(),
                                rk[b].numpy(), rv[b].numpy(), int(ctx[b]), DC["block"],
                                DC["window"], scale, gate=Gd[b].numpy())
        for r in res:
            assert np.abs(r[3][b] - ref).max() <= 1e-12
