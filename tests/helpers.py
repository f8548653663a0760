"""Shared plumbing for the GPU parity tests: move seeded inputs to the device,
call the C ABI through the binding, and compare with the oracle."""
import numpy as np
import torch

# Acceptance bars: fp32 path max-abs <= 1e-4; bf16 path relative L2 <= 1e-2 and max-abs <= 3e-2.
TOL_F32_MAXABS = 1e-4
TOL_BF16_RELL2 = 1e-2
TOL_BF16_MAXABS = 3e-2


def check_close(got, ref, dtype: str, what: str = ""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    mask = ~np.isnan(ref)
    assert np.all(np.isfinite(got[mask])), f"{what}: non-finite GPU output"
    d = np.abs(got[mask] - ref[mask])
    maxabs = float(d.max()) if d.size else 0.0
    if dtype == "f32":
        assert maxabs <= TOL_F32_MAXABS, f"{what}: max-abs {maxabs:.3e} > {TOL_F32_MAXABS}"
        return dict(maxabs=maxabs)
    rel = float(np.linalg.norm(got[mask] - ref[mask]) / max(np.linalg.norm(ref[mask]), 1e-30))
    assert rel <= TOL_BF16_RELL2, f"{what}: rel-L2 {rel:.3e} > {TOL_BF16_RELL2}"
    assert maxabs <= TOL_BF16_MAXABS, f"{what}: max-abs {maxabs:.3e} > {TOL_BF16_MAXABS}"
    return dict(maxabs=maxabs, rel_l2=rel)


def dims_of(mla, d, block_size, layout=0):
    return mla.make_dims(d.n_heads, d.d_c, d.d_rope, d.d_nope, d.d_v, d.d_model, block_size, d.dtype,
                         rope_base=d.rope_base, rms_eps=d.rms_eps, cache_layout=layout)


def tiled_ok(d, block_size):
    """The tiled page layout needs bf16, 64-token pages inside blocks and 64-dim chunks."""
    return d.dtype == "bf16" and block_size % 64 == 0 and (d.d_c + d.d_rope) % 64 == 0


def device_pool(mla, d, block_size, pool_rows_cpu, layout):
    """The latent pool on the device in the requested layout: (c_kv, k_pe, keepalive)."""
    rows = pool_rows_cpu.cuda()
    if layout == 0:
        return rows, rows[:, d.d_c:], rows
    tiled = torch.empty_like(rows)
    mla.mla_cache_pack(dims_of(mla, d, block_size, 1), rows, tiled)
    return tiled, tiled, tiled


def to_dev(inp, keys):
    return {k: inp[k].cuda() for k in keys}


def gpu_decode(mla, inp, latent=False, status=None, layout=None):
    """Run mla_decode (or mla_decode_latent) on the device; returns CPU (out, lse, dev_status).

    layout: 0 row pool, 1 tiled page pool; default tiled where the shape allows it."""
    d = inp["dims"]
    bs = inp["block_size"]
    if layout is None:
        layout = 1 if tiled_ok(d, bs) else 0
    dims = dims_of(mla, d, bs, layout)
    dev = to_dev(inp, ["q_nope", "q_pe", "block_table", "seqlens", "w_uk", "w_uv"])
    B, n_q, H = inp["q_nope"].shape[:3]
    max_seqlen = int(inp["seqlens"].max())
    c_kv, k_pe, _keep = device_pool(mla, d, bs, inp["pool"], layout)
    width = d.d_c if latent else d.d_v
    out = torch.full((B, n_q, H, width), float("nan"), dtype=d.torch_dtype, device="cuda")
    lse = torch.full((B, n_q, H), float("nan"), dtype=torch.float32, device="cuda")
    ws = mla.alloc_workspace(mla.mla_decode_workspace_size(dims, B, n_q, max_seqlen))
    st = torch.zeros(1, dtype=torch.int32, device="cuda") if status is None else status
    bt = dev["block_table"] if inp["case"].paged else None
    if latent:
        mla.mla_decode_latent(dims, dev["q_nope"], dev["q_pe"], c_kv, k_pe, bt, inp["max_blocks_per_seq"],
                              inp["num_blocks"], dev["seqlens"], max_seqlen, dev["w_uk"], out, lse, ws, st)
    else:
        mla.mla_decode(dims, dev["q_nope"], dev["q_pe"], c_kv, k_pe, bt, inp["max_blocks_per_seq"],
                       inp["num_blocks"], dev["seqlens"], max_seqlen, dev["w_uk"], dev["w_uv"], out, lse, ws, st)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy(), int(st.item())
