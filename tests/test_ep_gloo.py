"""Expert parallelism's exchange protocol on gloo ranks (CPU).

``ep_forward`` runs with the experts split across 2 or 4 ranks; a backend
built from the oracle stands in for the kernels (route, permutation, the
experts on grouped rows, the shared expert, the restore), so that what is
tested is the split, the two all-to-alls and the bookkeeping around them.
Each rank's output must equal the single-process oracle block on its own
tokens.  Cases: uneven token counts, a rank with no tokens, and routing forced
onto one rank's experts (the other ranks receive no rows).
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from routed_moe_layer_b200.dist import ep_send_counts, ep_split


def test_ep_split_and_send_counts():
    assert ep_split(128, 4, 0) == (0, 32) and ep_split(128, 4, 3) == (96, 32)
    with pytest.raises(ValueError):
        ep_split(10, 4, 0)
    offs = [0, 2, 2, 5, 9, 9, 9, 12, 15]  # E = 8
    assert ep_send_counts(offs, 8, 2) == [9, 6]
    assert ep_send_counts(offs, 8, 4) == [2, 7, 0, 6]
    assert sum(ep_send_counts(offs, 8, 8)) == offs[-1]


class OracleBackend:
    """The compute steps of ep_forward written with the oracle (float64, CPU)."""

    weight_dtype = torch.float64

    def __init__(self, ocfg):
        self.ocfg = ocfg

    def route(self, x, Wr, bias, cfg):
        import oracle
        ids, w, _, _ = oracle.route(x.numpy(), Wr.numpy(), bias.numpy(), self.ocfg)
        return torch.from_numpy(ids.astype(np.int32)), torch.from_numpy(w)

    def permute(self, ids, w, x, cfg):
        import oracle
        T, k = ids.shape
        offsets, row_of, tok_of = oracle.permutation(ids.numpy(), cfg.E)
        entry_of_row = np.empty(T * k, dtype=np.int64)
        entry_of_row[row_of] = np.arange(T * k)
        return dict(expert_offsets=torch.from_numpy(offsets.astype(np.int32)),
                    row_of=torch.from_numpy(row_of.astype(np.int32)),
                    tok_of=torch.from_numpy(tok_of.astype(np.int32)),
                    w_of=torch.from_numpy(w.numpy().reshape(-1)[entry_of_row].copy()),
                    xp=torch.from_numpy(x.numpy()[tok_of]))

    def rows_expert_ids(self, offsets, E):
        o = offsets.numpy()
        return torch.from_numpy(np.repeat(np.arange(E), np.diff(o)).astype(np.int32))

    def expert_rows(self, xr, offsets, w13, w2, row_dest, row_w, y_rows):
        import oracle
        o = offsets.numpy()
        y = np.zeros((y_rows, xr.shape[1]))
        for g in range(len(o) - 1):
            rows = np.arange(o[g], o[g + 1])
            if rows.size:
                y[row_dest.numpy()[rows]] = row_w.numpy()[rows][:, None] * oracle.swiglu_mlp(
                    xr.numpy()[rows], w13[g].numpy(), w2[g].numpy())
        return torch.from_numpy(y)

    def dense_ffn(self, x, w13, w2):
        import oracle
        return torch.from_numpy(oracle.dense_ffn(x.numpy(), w13.numpy(), w2.numpy()))

    def combine_rows(self, y, row_of, top_k, shared, residual):
        ro = row_of.numpy().reshape(-1, top_k)
        out = np.zeros((ro.shape[0], y.shape[1]))
        for j in range(top_k):
            ok = ro[:, j] >= 0
            out[ok] += y.numpy()[ro[ok, j]]
        if shared is not None:
            out += shared.numpy()
        if residual is not None:
            out += residual.numpy()
        return torch.from_numpy(out)

    def to_host(self, t):
        return [int(v) for v in t.tolist()]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, tokens, forced, result_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from routed_moe_layer_b200 import inputs
        from routed_moe_layer_b200.dist import ep_forward, ep_split, rank_token_seed
        from routed_moe_layer_b200.ops import BlockConfig
        from tests import parity
        H, E, I, k = 64, 16, 32, 4
        cfg = BlockConfig(T=tokens[rank], H=H, E=E, I=I, I_shared=I, top_k=k, n_group=4,
                          topk_group=2)
        wts = inputs.make_weights(H, 7, E=E, I=I, I_shared=I, wr_std=H ** -0.5,
                                  w13_std=H ** -0.5, w2_std=I ** -0.5)
        if forced:  # every token picks experts 0..3: all rows go to rank 0
            wts["bias"][:4] = 100.0
        x = inputs.make_tokens(tokens[rank], H, rank_token_seed(7, rank))
        d = {n: (None if v is None else v.double()) for n, v in wts.items()}
        xd = x.double()
        base, el = ep_split(E, world, rank)
        ocfg = parity.oracle_cfg(cfg)
        out = ep_forward(xd, d["Wr"], d["bias"], d["w13"][base:base + el],
                         d["w2"][base:base + el], d["ws13"], d["ws2"], cfg,
                         backend=OracleBackend(ocfg))
        if tokens[rank] > 0:
            ref, _, _, _ = oracle.moe_forward(xd.numpy(), d["Wr"].numpy(), d["bias"].numpy(),
                                              d["w13"].numpy(), d["w2"].numpy(),
                                              d["ws13"].numpy(), d["ws2"].numpy(), ocfg)
            err = float(np.abs(out.numpy() - ref).max())
        else:
            err = 0.0 if out.shape == (0, H) else float("inf")
        np.save(os.path.join(result_dir, f"r{rank}.npy"), np.array([err]))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("tokens,forced", [
    ((37, 53), False),
    ((29, 0), False),
    ((41, 23), True),
    ((11, 0, 19, 30), False),
])
def test_ep_ranks_equal_the_single_process_block(tmp_path, tokens, forced):
    world = len(tokens)
    mp.start_processes(_worker, args=(world, _free_port(), tokens, forced, str(tmp_path)),
                       nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        err = float(np.load(str(tmp_path / f"r{r}.npy"))[0])
        assert err < 1e-9, (r, err)
