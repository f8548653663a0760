"""mla_decode_noalloc: the decode entry point for callers that cannot allocate
device memory (for example code embedded in a runtime that owns every device
allocation).  It must give the same results as mla_decode with a caller
workspace, call after call, while the library's static scratch is reused.

This file is collected last so that a stop-at-first-failure run has already
run every other test before it."""
import numpy as np
import pytest
import torch

import oracle
from workloads import DECODE_CASES, make_decode_inputs
from helpers import check_close, dims_of, gpu_decode

pytestmark = pytest.mark.gpu


def _noalloc(mla, inp):
    d = inp["dims"]
    dims = dims_of(mla, d, inp["block_size"])
    dev = {k: inp[k].cuda() for k in ("q_nope", "q_pe", "pool", "block_table", "seqlens", "w_uk", "w_uv")}
    B, n_q, H = inp["q_nope"].shape[:3]
    out = torch.full((B, n_q, H, d.d_v), float("nan"), dtype=d.torch_dtype, device="cuda")
    lse = torch.full((B, n_q, H), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pool = dev["pool"]
    bt = dev["block_table"] if inp["case"].paged else None
    mla.mla_decode_noalloc(dims, dev["q_nope"], dev["q_pe"], pool, pool[:, d.d_c:], bt, inp["max_blocks_per_seq"],
                           inp["num_blocks"], dev["seqlens"], int(inp["seqlens"].max()), dev["w_uk"], dev["w_uv"],
                           out, lse, st)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy(), int(st.item())


@pytest.mark.parametrize("name", ["small_v2lite_bf16", "small_f32_nq2"])
def test_noalloc_matches_workspace_entry_point_twice(lib, name):
    inp = make_decode_inputs(DECODE_CASES[name])
    ref, ref_lse, st = gpu_decode(lib, inp)
    assert st == 0
    # The fp64 oracle on the same inputs, so the no-allocation path is held to the same bar as mla_decode.
    o_ref, o_lse = oracle.decode(inp["dims"], inp["q_nope"], inp["q_pe"], inp["pool"], inp["block_table"],
                                 inp["block_size"], inp["seqlens"], inp["w_uk"], inp["w_uv"])
    tol = 1e-4 if inp["dims"].dtype == "f32" else 3e-2
    for _ in range(2):            # the second call reuses the scratch the first one left behind
        out, lse, st = _noalloc(lib, inp)
        assert st == 0
        check_close(out, ref, inp["dims"].dtype, name + " noalloc vs mla_decode")
        assert np.max(np.abs(lse - ref_lse)) <= tol
        check_close(out, o_ref, inp["dims"].dtype, name + " noalloc vs oracle")
        assert np.max(np.abs(lse - o_lse)) <= tol


def test_noalloc_rejects_shapes_beyond_its_scratch(lib):
    """The V3 batch-64 x 4096 step needs far more than 16 MiB of scratch: refused before launch."""
    case = DECODE_CASES["v3_bf16"]
    d = case.dims
    dims = dims_of(lib, d, case.block_size)
    need = lib.mla_decode_workspace_size(dims, case.batch, case.n_q, 4096)
    assert need > lib.NOALLOC_SCRATCH_BYTES
    q = torch.zeros((case.batch, 1, d.n_heads, d.d_nope), dtype=torch.bfloat16, device="cuda")
    qp = torch.zeros((case.batch, 1, d.n_heads, d.d_rope), dtype=torch.bfloat16, device="cuda")
    pool = torch.zeros((64, d.d_c + d.d_rope), dtype=torch.bfloat16, device="cuda")
    sl = torch.full((case.batch,), 4096, dtype=torch.int32, device="cuda")
    w = torch.zeros((d.n_heads, d.d_c, d.d_nope), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((case.batch, 1, d.n_heads, d.d_v), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.MlaError) as e:
        lib.mla_decode_noalloc(dims, q, qp, pool, pool[:, d.d_c:], None, 64, 4096, sl, 4096, w, w, out, None)
    assert e.value.code == -7
