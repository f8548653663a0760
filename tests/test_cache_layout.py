"""GPU checks of the tiled page layout: pack/unpack is a bit-exact permutation
with the documented element positions, and the append writes the same bytes
into a tiled pool as into a row pool."""
import numpy as np
import pytest
import torch

from workloads import Dims, V3, make_append_inputs
from helpers import dims_of

pytestmark = pytest.mark.gpu


def _tiled_position(r, d, W):
    """Byte offset of element (row r, dim d) in the tiled layout, from its definition."""
    page, t = divmod(r, 64)
    c, rest = divmod(d, 64)
    g, e = divmod(rest, 8)
    return page * W * 128 + c * 8192 + t * 128 + 16 * (g ^ (t % 8)) + 2 * e


def test_pack_unpack_roundtrip_and_positions(lib):
    d = Dims(**V3)
    W = d.d_c + d.d_rope
    rows = torch.randn(4 * 64, W).to(torch.bfloat16).cuda()
    dims = dims_of(lib, d, 64, 1)
    tiled = torch.empty_like(rows)
    lib.mla_cache_pack(dims, rows, tiled)
    back = torch.full_like(rows, float("nan"))
    lib.mla_cache_unpack(dims, tiled, back)
    torch.cuda.synchronize()
    assert torch.equal(back.view(torch.int16), rows.view(torch.int16))
    flat = tiled.view(torch.int16).flatten().cpu().numpy()
    src = rows.view(torch.int16).cpu().numpy()
    rng = np.random.default_rng(0)
    for _ in range(2000):
        r, dd = int(rng.integers(rows.shape[0])), int(rng.integers(W))
        assert flat[_tiled_position(r, dd, W) // 2] == src[r, dd]


@pytest.mark.parametrize("block", [64, 128])
def test_append_tiled_equals_rows(lib, block):
    d = Dims(**V3)
    seqlens = torch.tensor([70, 200, 129], dtype=torch.int32)
    inp = make_append_inputs(d, 29, seqlens, block, True, seed=77)
    dev = {k: inp[k].cuda() for k in ("h", "w_dkv", "w_kr", "gamma", "seq_idx", "pos", "block_table")}
    nrows = inp["num_blocks"] * block
    outs = []
    for layout in (0, 1):
        pool = torch.full((nrows, d.d_c + d.d_rope), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        dims = dims_of(lib, d, block, layout)
        lib.mla_append_latent(dims, dev["h"], dev["w_dkv"], dev["w_kr"], dev["gamma"], dev["seq_idx"], dev["pos"],
                              pool, pool[:, d.d_c:] if layout == 0 else pool, dev["block_table"], 3,
                              inp["max_blocks_per_seq"], inp["num_blocks"], st)
        if layout == 1:
            rows = torch.empty_like(pool)
            lib.mla_cache_unpack(dims, pool, rows)
            pool = rows
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        outs.append(pool.view(torch.int16).cpu())
    assert torch.equal(outs[0], outs[1])
