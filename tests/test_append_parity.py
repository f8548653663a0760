"""GPU parity of mla_append_latent: content against the oracle, position and
bytes bit-exact between a paged and a contiguous table."""
import numpy as np
import pytest
import torch

import oracle
from workloads import Dims, V3, make_append_inputs
from helpers import check_close, dims_of

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_f32": (Dims(8, 64, 16, 32, 32, 256, "f32"), 13, (9, 40, 33), 16),
    "v3_bf16_decode": (Dims(**V3), 64, tuple([4096] * 64), 64),
    "v3_bf16_ragged": (Dims(**V3), 37, (1, 64, 65, 300, 129), 64),
}


def _run(mla, inp, paged: bool, pool_rows: int, dims_, mma: bool = True):
    d = inp["dims"]
    dev = {k: inp[k].cuda() for k in ("h", "w_dkv", "w_kr", "gamma", "seq_idx", "pos", "block_table")}
    pool = torch.full((pool_rows, d.d_c + d.d_rope), float("nan"), dtype=d.torch_dtype, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    bt = dev["block_table"] if paged else None
    nws = mla.mla_append_workspace_size(dims_, inp["h"].shape[0]) if mma else 0
    ws = mla.alloc_workspace(nws) if nws else None
    mla.mla_append_latent(dims_, dev["h"], dev["w_dkv"], dev["w_kr"], dev["gamma"], dev["seq_idx"], dev["pos"],
                          pool, pool[:, d.d_c:], bt, inp["seqlens"].numel(), inp["max_blocks_per_seq"],
                          pool_rows // inp["block_size"], st, workspace=ws)
    torch.cuda.synchronize()
    return pool.cpu(), int(st.item())


@pytest.mark.parametrize("mma", [True, False])
@pytest.mark.parametrize("name", list(CASES))
def test_append_content_and_layout(lib, name, mma):
    """mma=True: tensor-core projection (bf16 shapes, with workspace); False: the CUDA-core kernel."""
    d, T, seqlens, bs = CASES[name]
    inp = make_append_inputs(d, T, torch.tensor(seqlens, dtype=torch.int32), bs, True, seed=300 + T)
    dims_ = dims_of(lib, d, bs)
    pool, st = _run(lib, inp, True, inp["num_blocks"] * bs, dims_, mma)
    assert st == 0
    c_ref, k_ref = oracle.append_latent(inp["h"], inp["w_dkv"], inp["w_kr"], inp["gamma"], inp["pos"],
                                        d.rms_eps, d.rope_base)
    bt = inp["block_table"]
    rows = [int(bt[b, p // bs]) * bs + p % bs for b, p in zip(inp["seq_idx"].tolist(), inp["pos"].tolist())]
    got = pool[rows].float().numpy()
    check_close(got[:, :d.d_c], c_ref, d.dtype, name + " c_KV")
    check_close(got[:, d.d_c:], k_ref, d.dtype, name + " k_pe")
    # Every other row is untouched (still the NaN sentinel).
    untouched = np.ones(pool.shape[0], dtype=bool)
    untouched[rows] = False
    assert torch.isnan(pool[torch.from_numpy(untouched)].float()).all()


@pytest.mark.parametrize("name", list(CASES))
def test_append_paged_equals_contiguous_bitwise(lib, name):
    d, T, seqlens, bs = CASES[name]
    inp = make_append_inputs(d, T, torch.tensor(seqlens, dtype=torch.int32), bs, True, seed=400 + T)
    dims_ = dims_of(lib, d, bs)
    mbps = inp["max_blocks_per_seq"]
    B = len(seqlens)
    paged, st1 = _run(lib, inp, True, inp["num_blocks"] * bs, dims_)
    contig, st2 = _run(lib, inp, False, B * mbps * bs, dims_)
    assert st1 == 0 and st2 == 0
    bt = inp["block_table"]
    for b, p in zip(inp["seq_idx"].tolist(), inp["pos"].tolist()):
        r_p = int(bt[b, p // bs]) * bs + p % bs
        r_c = b * mbps * bs + p
        assert torch.equal(paged[r_p].view(torch.int16 if d.dtype == "bf16" else torch.int32),
                           contig[r_c].view(torch.int16 if d.dtype == "bf16" else torch.int32))


def test_append_bad_position_is_reported(lib):
    d, T, seqlens, bs = CASES["tiny_f32"]
    inp = make_append_inputs(d, T, torch.tensor(seqlens, dtype=torch.int32), bs, True, seed=7)
    inp["pos"] = inp["pos"].clone()
    inp["pos"][3] = inp["max_blocks_per_seq"] * bs + 1
    pool, st = _run(lib, inp, True, inp["num_blocks"] * bs, dims_of(lib, d, bs))
    assert st == -6
