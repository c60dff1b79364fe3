"""Multi-rank path on CPU: two gloo ranks each compute their own share of the streams (the fp64
oracle stands in for the GPU kernel on a GPU-less host), with no collective on the data path;
gathering the shares reproduces the single-process result, and the timing reduction takes the
max over ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, outdir):
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    from oracle import ttt_oracle as orc
    from weight_linear_attention_ttt_b200 import inputs as inp
    from weight_linear_attention_ttt_b200.shard import (max_over_ranks, shard_columns,
                                                        shard_streams)

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        # dual form: shard (b,h) streams along the batch dimension
        x = inp.dual_or_assoc_inputs(4, 2, 64, 16, seed=3, device="cpu", normalise=("K", "V"))
        mine = shard_streams(x, rank, world)
        O, W = orc.dual_form(mine["Q"].float().numpy(), mine["K"].float().numpy(),
                             mine["V"].float().numpy(), mine["eta"].numpy(),
                             mine["W0"].numpy(), 16)
        np.save(os.path.join(outdir, f"dual_O_{rank}.npy"), O)
        np.save(os.path.join(outdir, f"dual_W_{rank}.npy"), W)
        # In-Place: shard output columns; Z is shared
        z = inp.inplace_inputs(64, 32, 24, seed=4, device="cpu", eta=0.05)
        zc = shard_columns(z, rank, world)
        Oi, Wi = orc.inplace_chunks(zc["Z"].float().numpy(), zc["Vhat"].float().numpy(),
                                    zc["W0"].float().numpy(), zc["eta"], 32)
        np.save(os.path.join(outdir, f"inp_O_{rank}.npy"), Oi)
        np.save(os.path.join(outdir, f"inp_W_{rank}.npy"), Wi)
        # timing reduction: max over ranks
        m = max_over_ranks(10.0 + rank)
        np.save(os.path.join(outdir, f"max_{rank}.npy"), np.array([m]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_without_data_collectives(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    from oracle import ttt_oracle as orc
    from weight_linear_attention_ttt_b200 import inputs as inp

    x = inp.dual_or_assoc_inputs(4, 2, 64, 16, seed=3, device="cpu", normalise=("K", "V"))
    O, W = orc.dual_form(x["Q"].float().numpy(), x["K"].float().numpy(), x["V"].float().numpy(),
                         x["eta"].numpy(), x["W0"].numpy(), 16)
    Og = np.concatenate([np.load(tmp_path / f"dual_O_{r}.npy") for r in range(world)])
    Wg = np.concatenate([np.load(tmp_path / f"dual_W_{r}.npy") for r in range(world)])
    np.testing.assert_array_equal(Og, O)
    np.testing.assert_array_equal(Wg, W)

    z = inp.inplace_inputs(64, 32, 24, seed=4, device="cpu", eta=0.05)
    Oi, Wi = orc.inplace_chunks(z["Z"].float().numpy(), z["Vhat"].float().numpy(),
                                z["W0"].float().numpy(), z["eta"], 32)
    Oig = np.concatenate([np.load(tmp_path / f"inp_O_{r}.npy") for r in range(world)], axis=1)
    Wig = np.concatenate([np.load(tmp_path / f"inp_W_{r}.npy") for r in range(world)], axis=1)
    np.testing.assert_allclose(Oig, Oi, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(Wig, Wi, rtol=1e-12, atol=1e-12)

    for r in range(world):
        assert float(np.load(tmp_path / f"max_{r}.npy")[0]) == 11.0


def _cp_worker(rank, world, port, outdir):
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    from oracle import ttt_oracle as orc
    from weight_linear_attention_ttt_b200 import inputs as inp
    from weight_linear_attention_ttt_b200.context_parallel import assoc_scan_fwd_cp
    from weight_linear_attention_ttt_b200.shard import split_range

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        B, H, T, d, C = 2, 2, 256, 8, 16
        x = inp.dual_or_assoc_inputs(B, H, T, d, seed=12, device="cpu", normalise=("Q", "K"),
                                     eta="sigmoid", w0="normal_0.02")
        t0, t1 = split_range(T // C, rank, world)
        sl = slice(t0 * C, t1 * C)
        Q, K, V = (x[k][:, :, sl].double() for k in ("Q", "K", "V"))
        eta = x["eta"][:, :, sl].double()
        S0 = x["W0"].double()

        def per_stream(fn, *args):
            outs = [[fn(*(a[b, h] for a in args)) for h in range(H)] for b in range(B)]
            return outs

        def state_fn(K_, V_, e_):
            res = per_stream(lambda k, v, e: orc.assoc_chunked_stream(k, k, v, e, None, C)[1],
                             K_.numpy(), V_.numpy(), e_.numpy())
            return torch.tensor(np.array(res))

        def scan_fn(Q_, K_, V_, e_, s_):
            res = per_stream(lambda q, k, v, e, s: orc.assoc_chunked_stream(q, k, v, e, s, C),
                             Q_.numpy(), K_.numpy(), V_.numpy(), e_.numpy(), s_.numpy())
            O = torch.tensor(np.array([[r[0] for r in row] for row in res]))
            S = torch.tensor(np.array([[r[1] for r in row] for row in res]))
            return O, S

        def prefix_fn(s0, inc, upto):
            return s0 + inc[:upto].sum(0)

        O, S_final = assoc_scan_fwd_cp(Q, K, V, eta, S0, C=C, state_fn=state_fn,
                                       scan_fn=scan_fn, prefix_fn=prefix_fn)
        np.save(os.path.join(outdir, f"cp_O_{rank}.npy"), O.numpy())
        np.save(os.path.join(outdir, f"cp_S_{rank}.npy"), S_final.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_assoc_scan_over_gloo_ranks(tmp_path, world):
    """Each rank owns a slice of the sequence; one all-gather of the slices' state increments
    and a prefix sum give every rank its starting state; the gathered outputs and the final
    state equal the sequential recurrence."""
    mp.start_processes(_cp_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    from oracle import ttt_oracle as orc
    from weight_linear_attention_ttt_b200 import inputs as inp

    x = inp.dual_or_assoc_inputs(2, 2, 256, 8, seed=12, device="cpu", normalise=("Q", "K"),
                                 eta="sigmoid", w0="normal_0.02")
    O, S = orc.assoc_scan(x["Q"].double().numpy(), x["K"].double().numpy(),
                          x["V"].double().numpy(), x["eta"].double().numpy(),
                          x["W0"].double().numpy())
    Og = np.concatenate([np.load(tmp_path / f"cp_O_{r}.npy") for r in range(world)], axis=2)
    np.testing.assert_allclose(Og, O, rtol=1e-10, atol=1e-12)
    for r in range(world):
        np.testing.assert_allclose(np.load(tmp_path / f"cp_S_{r}.npy"), S, rtol=1e-10,
                                   atol=1e-12)


def _dual_cp_worker(rank, world, port, outdir):
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import numpy as np
    import torch
    import torch.distributed as dist

    from oracle import ttt_oracle as orc
    from weight_linear_attention_ttt_b200 import inputs as inp
    from weight_linear_attention_ttt_b200.context_parallel import dual_form_fwd_cp
    from weight_linear_attention_ttt_b200.shard import split_range

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        B, H, T, d, C = 2, 2, 256, 8, 16
        x = inp.dual_or_assoc_inputs(B, H, T, d, seed=13, device="cpu", normalise=("K", "V"),
                                     eta="sigmoid", w0="normal_0.02")
        t0, t1 = split_range(T // C, rank, world)
        sl = slice(t0 * C, t1 * C)
        Q, K, V = (x[k][:, :, sl].double() for k in ("Q", "K", "V"))
        eta = x["eta"][:, :, sl].double()
        W0 = x["W0"].double()

        def per_stream(fn, *args):
            return [[fn(*(a[b, h] for a in args)) for h in range(H)] for b in range(B)]

        def maps_fn(K_, V_, e_):
            res = per_stream(lambda k, v, e: orc.dual_segment_maps_stream(k, v, e, C),
                             K_.numpy(), V_.numpy(), e_.numpy())
            A = torch.tensor(np.array([[r[0] for r in row] for row in res]))
            Bm = torch.tensor(np.array([[r[1] for r in row] for row in res]))
            return A, Bm

        def scan_fn(Q_, K_, V_, e_, w_):
            res = per_stream(lambda q, k, v, e, w: orc.dual_form_stream(q, k, v, e, w, C),
                             Q_.numpy(), K_.numpy(), V_.numpy(), e_.numpy(), w_.numpy())
            O = torch.tensor(np.array([[r[0] for r in row] for row in res]))
            W = torch.tensor(np.array([[r[1] for r in row] for row in res]))
            return O, W

        def fold_fn(w0, A_all, B_all, upto):
            W = w0.clone()
            for m in range(upto):
                W = A_all[m] @ W + B_all[m]
            return W

        O, W_final = dual_form_fwd_cp(Q, K, V, eta, W0, C=C, maps_fn=maps_fn, scan_fn=scan_fn,
                                      fold_fn=fold_fn)
        np.save(os.path.join(outdir, f"dcp_O_{rank}.npy"), O.numpy())
        np.save(os.path.join(outdir, f"dcp_W_{rank}.npy"), W_final.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_dual_form_over_gloo_ranks(tmp_path, world):
    """Each rank owns a slice of the sequence; one all-gather of the slices' affine maps and an
    ordered fold give every rank its start state; the gathered outputs and the final state equal
    the sequential dual form."""
    mp.start_processes(_dual_cp_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    from oracle import ttt_oracle as orc
    from weight_linear_attention_ttt_b200 import inputs as inp

    x = inp.dual_or_assoc_inputs(2, 2, 256, 8, seed=13, device="cpu", normalise=("K", "V"),
                                 eta="sigmoid", w0="normal_0.02")
    O, W = orc.dual_form(x["Q"].double().numpy(), x["K"].double().numpy(),
                         x["V"].double().numpy(), x["eta"].double().numpy(),
                         x["W0"].double().numpy(), 16)
    Og = np.concatenate([np.load(tmp_path / f"dcp_O_{r}.npy") for r in range(world)], axis=2)
    np.testing.assert_allclose(Og, O, rtol=1e-10, atol=1e-12)
    for r in range(world):
        np.testing.assert_allclose(np.load(tmp_path / f"dcp_W_{r}.npy"), W, rtol=1e-10,
                                   atol=1e-12)
