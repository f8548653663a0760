"""Host logic of the multi-GPU decode (mla_latent_kv_40_b200.sharded) on CPU.

The shard arithmetic is checked exhaustively; the exact merge of key-range
partials is pinned against the fp64 oracle's decode over all keys; and the
all-gather of partials runs on two gloo ranks (127.0.0.1), each rank holding
the oracle's partial of its own key range."""
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch

import oracle
from workloads import DECODE_CASES, make_decode_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _sharded():
    sys.path.insert(0, ROOT)
    import importlib.util
    spec = importlib.util.spec_from_file_location("sharded", os.path.join(ROOT, "mla_latent_kv_40_b200", "sharded.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("batch,world", [(64, 1), (64, 8), (7, 3), (3, 8), (128, 5)])
def test_batch_shard_partitions_the_batch(batch, world):
    sh = _sharded()
    slices = [sh.batch_shard(batch, world, r) for r in range(world)]
    assert slices[0][0] == 0 and slices[-1][1] == batch
    for (a0, a1), (b0, b1) in zip(slices, slices[1:]):
        assert a1 == b0
    sizes = [b - a for a, b in slices]
    assert max(sizes) - min(sizes) <= 1


@pytest.mark.parametrize("max_seqlen,world", [(131072, 4), (131072, 8), (300, 4), (64, 3), (4096, 2), (100, 1)])
def test_kv_shard_ranges_cover_the_keys(max_seqlen, world):
    sh = _sharded()
    rng = sh.kv_shard_ranges(max_seqlen, world)
    assert len(rng) == world and rng[0][0] == 0 and rng[-1][1] == max_seqlen
    for (a0, a1), (b0, b1) in zip(rng, rng[1:]):
        assert a1 == b0 or (a0 == a1 and b0 == a0) or a1 == b0
    for b, e in rng:
        assert b % 64 == 0 and e >= b
    covered = sum(e - b for b, e in rng)
    assert covered == max_seqlen


def _partials(inp, ranges, heads=None):
    """The oracle's partial of each key range: the decode over that range's visible keys, with
    W_UV = I (the latent), as (o [N, B, n_q, H, d_c], lse [N, B, n_q, H]); empty ranges give
    (0, -inf).  With `heads`, only those heads are computed (the others stay NaN)."""
    d = inp["dims"]
    B, n_q, H = inp["q_nope"].shape[:3]
    sl = inp["seqlens"].numpy()
    eye = np.broadcast_to(np.eye(d.d_c), (H, d.d_c, d.d_c))
    import dataclasses
    dl = dataclasses.replace(d, d_v=d.d_c)
    heads = list(range(H)) if heads is None else list(heads)
    o = np.zeros((len(ranges), B, n_q, H, d.d_c))
    lse = np.full((len(ranges), B, n_q, H), -np.inf)
    skip = [x for x in range(H) if x not in heads]
    o[:, :, :, skip] = np.nan
    lse[:, :, :, skip] = np.nan
    for r, (k0, k1) in enumerate(ranges):
        for b in range(B):
            for j in range(n_q):
                p = int(sl[b]) - n_q + j
                toks = list(range(k0, min(k1, p + 1)))
                if not toks:
                    continue
                sel = np.full((B, n_q, len(toks)), -1)
                sel[b, j] = toks
                picks = [(b, j, s) for s in heads]
                ob, lb = oracle.decode_sparse(dl, inp["q_nope"], inp["q_pe"], inp["pool"], inp["block_table"],
                                              inp["block_size"], inp["seqlens"], sel, inp["w_uk"], eye, picks=picks)
                o[r, b, j, heads] = ob[b, j, heads]
                lse[r, b, j, heads] = lb[b, j, heads]
    return o, lse


def _merge(o, lse, w_uv):
    """LSE = ln sum_r exp(lse_r), o_lat = sum_r exp(lse_r - LSE) o_r, out^(s) = o_lat^(s) W_UV^(s)."""
    m = np.max(lse, axis=0)
    w = np.exp(lse - m[None])
    LSE = m + np.log(np.sum(w, axis=0))
    o_lat = np.sum(np.exp(lse - LSE[None])[..., None] * o, axis=0)
    out = np.einsum("bjsc,scv->bjsv", o_lat, np.asarray(w_uv, dtype=np.float64))
    return out, LSE


@pytest.mark.parametrize("world", [2, 3, 4])
def test_merge_of_key_range_partials_is_the_full_decode(world):
    """Merging the partials of disjoint key ranges by their log-sum-exps reproduces the decode over
    all keys, to fp64 rounding (case with two causal query tokens and ragged lengths)."""
    sh = _sharded()
    inp = make_decode_inputs(DECODE_CASES["small_f32_nq2"])
    ranges = sh.kv_shard_ranges(int(inp["seqlens"].max()), world, align=16)
    o, lse = _partials(inp, ranges)
    out, LSE = _merge(o, lse, inp["w_uv"].double().numpy())
    ref, ref_lse = oracle.decode(inp["dims"], inp["q_nope"], inp["q_pe"], inp["pool"], inp["block_table"],
                                 inp["block_size"], inp["seqlens"], inp["w_uk"], inp["w_uv"])
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(LSE, ref_lse, rtol=1e-12)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_rank(rank, world, port, out_path):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime

    import torch.distributed as dist
    import test_sharding as T
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    sh = T._sharded()
    inp = make_decode_inputs(DECODE_CASES["small_f32_nq2"])
    ranges = sh.kv_shard_ranges(int(inp["seqlens"].max()), world, align=16)
    o, lse = T._partials(inp, [ranges[rank]])           # this rank's own key range only
    o_all, l_all = sh.gather_partials(torch.from_numpy(o[0]), torch.from_numpy(lse[0]))
    out, LSE = T._merge(o_all.numpy(), l_all.numpy(), inp["w_uv"].double().numpy())
    dist.barrier()
    dist.destroy_process_group()
    np.save(out_path, out)


def test_split_kv_gather_over_two_gloo_ranks(tmp_path):
    """Each of two ranks computes the partial of its key range; after the all-gather both ranks
    hold every partial and their merge is the full decode."""
    import torch.multiprocessing as mp
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_gloo_rank, args=(r, 2, port, str(tmp_path / f"r{r}.npy"))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    inp = make_decode_inputs(DECODE_CASES["small_f32_nq2"])
    ref, _ = oracle.decode(inp["dims"], inp["q_nope"], inp["q_pe"], inp["pool"], inp["block_table"],
                           inp["block_size"], inp["seqlens"], inp["w_uk"], inp["w_uv"])
    for r in range(2):
        np.testing.assert_allclose(np.load(tmp_path / f"r{r}.npy"), ref, rtol=1e-11, atol=1e-12)
