"""CPU checks of the C ABI boundary: the library loads without a GPU, exports
every symbol include/mla.h declares, and rejects bad arguments on the host
before anything is launched."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "mla.h")).read()
    return sorted(set(re.findall(r"MLA_API\s+(?:const\s+char\s*\*|int)\s*(mla_\w+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for want in ("mla_append_latent", "mla_decode_workspace_size", "mla_decode", "mla_prefill",
                 "mla_prefill_workspace_size", "mla_status_string", "mla_absorb_q", "mla_decode_latent",
                 "mla_cache_pack", "mla_cache_unpack"):
        assert want in names


def test_library_exports_every_declared_symbol():
    import mla_latent_kv_40_b200 as mla
    lib = ctypes.CDLL(mla.LIB_PATH)
    for n in _declared():
        assert hasattr(lib, n), n


def test_status_strings():
    import mla_latent_kv_40_b200 as mla
    for code in range(-7, 1):
        assert mla.mla_status_string(code) and "unknown" not in mla.mla_status_string(code)
    assert "unknown" in mla.mla_status_string(-99)


def _prototypes():
    """name -> list of parameter type strings, parsed from include/mla.h."""
    src = open(os.path.join(ROOT, "include", "mla.h")).read()
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    out = {}
    for m in re.finditer(r"MLA_API\s+(?:const\s+char\s*\*|int)\s*(mla_\w+)\s*\(([^)]*)\)", src):
        params = [" ".join(p.split()) for p in m.group(2).split(",")]
        types = []
        for p in params:
            p = re.sub(r"\b\w+$", "", p).strip()         # drop the parameter name
            types.append(p.replace(" *", "*").replace("* ", "*"))
        out[m.group(1)] = types
    return out


def _ctype_of(c):
    """The ctypes class a C parameter type must be marshalled as (width matters on the stack)."""
    if c.endswith("*") or c == "mla_stream_t":
        return "ptr"
    return {"int": ctypes.c_int, "size_t": ctypes.c_size_t, "int64_t": ctypes.c_int64,
            "long long": ctypes.c_longlong}[c]


def test_binding_argtypes_match_header_prototypes():
    """Every entry point is called with declared argument types of the right count and width
    (an undeclared 64-bit argument passed on the stack arrives with a garbage upper half)."""
    import mla_latent_kv_40_b200 as mla
    protos = _prototypes()
    assert set(protos) == set(_declared())
    for name, ctypes_list in protos.items():
        fn = getattr(mla._lib, name)
        assert fn.argtypes is not None, name
        assert len(fn.argtypes) == len(ctypes_list), (name, len(fn.argtypes), len(ctypes_list))
        for i, (c, got) in enumerate(zip(ctypes_list, fn.argtypes)):
            want = _ctype_of(c)
            if want == "ptr":
                assert got is ctypes.c_void_p or issubclass(got, ctypes._Pointer), (name, i, c, got)
            else:
                assert issubclass(got, ctypes._SimpleCData) and ctypes.sizeof(got) == ctypes.sizeof(want), \
                    (name, i, c, got)


def test_dims_struct_matches_header_layout():
    import mla_latent_kv_40_b200 as mla
    assert ctypes.sizeof(mla.mla_dims) == 14 * 4


def _lib():
    import mla_latent_kv_40_b200 as mla
    return mla, mla._lib


def test_host_validation_rejects_bad_arguments():
    mla, lib = _lib()
    d = mla.make_dims(8, 64, 16, 32, 32, 256, 64, "f32")
    n = ctypes.c_size_t(0)
    assert lib.mla_decode_workspace_size(ctypes.byref(d), 0, 1, 10, ctypes.byref(n)) == -1
    assert lib.mla_decode_workspace_size(ctypes.byref(d), 1, 2, 1, ctypes.byref(n)) == -1   # max_seqlen < n_q
    assert lib.mla_decode_workspace_size(ctypes.byref(d), 1, 1, 10, None) == -1
    big = mla.make_dims(200, 64, 16, 32, 32, 256, 64, "f32")
    assert lib.mla_decode_workspace_size(ctypes.byref(big), 1, 2, 10, ctypes.byref(n)) == -2  # n_q*H > 256
    odd = mla.make_dims(8, 64, 15, 32, 32, 256, 64, "f32")
    assert lib.mla_decode_workspace_size(ctypes.byref(odd), 1, 1, 10, ctypes.byref(n)) == -1  # odd d_rope
    bad = mla.make_dims(8, 64, 16, 32, 32, 256, 64, "f32", ckv_stride=10)
    assert lib.mla_decode_workspace_size(ctypes.byref(bad), 1, 1, 10, ctypes.byref(n)) == -1  # stride < d_c
    assert lib.mla_decode_workspace_size(ctypes.byref(d), 1, 1, 10, ctypes.byref(n)) == 0 and n.value > 0
    P = ctypes.c_void_p
    fake = P(0x1000)
    # Missing pointers are caught before any launch.
    rc = lib.mla_decode(ctypes.byref(d), 1, 1, None, fake, fake, fake, None, 4, 4, fake, 10, fake, fake, fake,
                        None, fake, ctypes.c_size_t(1 << 20), None, None)
    assert rc == -1
    # Workspace too small / misaligned.
    rc = lib.mla_decode(ctypes.byref(d), 1, 1, fake, fake, fake, fake, None, 4, 4, fake, 10, fake, fake, fake,
                        None, fake, ctypes.c_size_t(16), None, None)
    assert rc == -3
    rc = lib.mla_decode(ctypes.byref(d), 1, 1, fake, fake, fake, fake, None, 4, 4, fake, 10, fake, fake, fake,
                        None, P(0x1001), ctypes.c_size_t(1 << 30), None, None)
    assert rc == -3
    # Table too short for max_seqlen.
    rc = lib.mla_decode(ctypes.byref(d), 1, 1, fake, fake, fake, fake, None, 1, 4, fake, 100, fake, fake, fake,
                        None, fake, ctypes.c_size_t(1 << 30), None, None)
    assert rc == -1
    # Append of zero tokens is a no-op that launches nothing.
    assert lib.mla_append_latent(ctypes.byref(d), 0, None, None, None, None, None, None, None, None, None,
                                 1, 1, 1, None, ctypes.c_size_t(0), None, None) == 0
    assert lib.mla_append_latent(ctypes.byref(d), 3, None, fake, fake, None, fake, fake, fake, fake, None,
                                 1, 1, 1, None, ctypes.c_size_t(0), None, None) == -1
    # The tensor-core append needs scratch for bf16 shapes only.
    assert lib.mla_append_workspace_size(ctypes.byref(d), 64, ctypes.byref(n)) == 0 and n.value == 0
    v3 = mla.make_dims(128, 512, 64, 128, 128, 7168, 64, "bf16")
    assert lib.mla_append_workspace_size(ctypes.byref(v3), 64, ctypes.byref(n)) == 0 and n.value > 0
    assert lib.mla_prefill_workspace_size(ctypes.byref(d), 1, 0, 10, ctypes.byref(n)) == -1
    # Tiled page pools: bf16 only, blocks of whole 64-token pages, rows of whole 64-dim chunks.
    t_ok = mla.make_dims(128, 512, 64, 128, 128, 7168, 64, "bf16", cache_layout=1)
    assert lib.mla_decode_workspace_size(ctypes.byref(t_ok), 2, 1, 100, ctypes.byref(n)) == 0
    for bad_t in (mla.make_dims(128, 512, 64, 128, 128, 7168, 64, "f32", cache_layout=1),
                  mla.make_dims(128, 512, 64, 128, 128, 7168, 32, "bf16", cache_layout=1),
                  mla.make_dims(128, 500, 64, 128, 128, 7168, 64, "bf16", cache_layout=1),
                  mla.make_dims(128, 512, 64, 128, 128, 7168, 64, "bf16", cache_layout=2)):
        assert lib.mla_decode_workspace_size(ctypes.byref(bad_t), 2, 1, 100, ctypes.byref(n)) == -1
    # Pack / unpack: row counts in whole pages, distinct buffers.
    assert lib.mla_cache_pack(ctypes.byref(t_ok), fake, P(0x100000000), 100, None) == -1
    assert lib.mla_cache_pack(ctypes.byref(t_ok), fake, fake, 64, None) == -1


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    """The product path has no fallback: a missing libmla.so is an ImportError."""
    import importlib.util
    import shutil
    pkg = tmp_path / "mla_latent_kv_40_b200"
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, "mla_latent_kv_40_b200", "__init__.py"), pkg / "__init__.py")
    spec = importlib.util.spec_from_file_location("mla_copy", pkg / "__init__.py")
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)


def test_decode_path_query():
    """mla_decode_path is host logic: the V3 and V2-Lite bf16 shapes take the tensor-core kernels,
    the fp32 shapes the CUDA-core kernels (no GPU needed)."""
    import mla_latent_kv_40_b200 as mla
    from workloads import DECODE_CASES
    for name, want in (("v3_bf16", mla.PATH_TCGEN05), ("v2lite_bf16", mla.PATH_TCGEN05),
                       ("v3_ragged_bf16", mla.PATH_TCGEN05), ("tiny_fp32", mla.PATH_CUDA_CORES),
                       ("small_f32_nq2", mla.PATH_CUDA_CORES)):
        case = DECODE_CASES[name]
        d = case.dims
        for layout in ((0, 1) if d.dtype == "bf16" else (0,)):
            dims = mla.make_dims(d.n_heads, d.d_c, d.d_rope, d.d_nope, d.d_v, d.d_model, case.block_size, d.dtype,
                                 cache_layout=layout)
            assert mla.mla_decode_path(dims, case.n_q) == want, (name, layout)
    with pytest.raises(mla.MlaError):
        mla.mla_decode_path(mla.make_dims(8, 64, 16, 32, 32, 256, 0, "f32"), 1)   # block_size 0


def test_bench_picks_the_traffic_entry_of_the_kernel_that_runs():
    """The bench's DRAM-traffic figure for the V3 batch-64 step is keyed by the tensor-core attention
    kernel's source file, which is what mla_decode_path reports for that shape."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import mla_latent_kv_40_b200 as mla
    from workloads import DECODE_CASES
    case = DECODE_CASES["v3_bf16"]
    d = case.dims
    dims = mla.make_dims(d.n_heads, d.d_c, d.d_rope, d.d_nope, d.d_v, d.d_model, case.block_size, d.dtype,
                         cache_layout=1)
    key = "decode_tc.cu" if mla.mla_decode_path(dims, case.n_q) == mla.PATH_TCGEN05 else "attn_simt.cu"
    assert key == "decode_tc.cu"
    assert key in bench._TRAFFIC_SOURCES


def test_sparse_decode_host_validation():
    """mla_decode_sparse rejects a missing selection and a non-positive topk before launching."""
    import mla_latent_kv_40_b200 as mla
    dims = mla.make_dims(128, 512, 64, 128, 128, 7168, 64, "bf16", cache_layout=1)
    n = ctypes.c_size_t(0)
    assert mla._lib.mla_decode_sparse_workspace_size(ctypes.byref(dims), 64, 1, 0, ctypes.byref(n)) == -1
    assert mla._lib.mla_decode_sparse_workspace_size(ctypes.byref(dims), 64, 1, 2048, ctypes.byref(n)) == 0
    # the gathered rows alone: 64 tokens x 2048 rows x 1152 bytes
    assert n.value >= 64 * 2048 * 1152
    fake = ctypes.c_void_p(256)
    rc = mla._lib.mla_decode_sparse(ctypes.byref(dims), 64, 1, fake, fake, fake, fake, None, 64, 4096, fake, 4096,
                                    None, 2048, fake, fake, fake, None, fake, n.value, None, None)
    assert rc == -1


def test_split_kv_host_validation():
    """mla_decode_partial needs a 64-aligned kv_begin, kv_end > kv_begin and an lse output;
    mla_merge_partials needs at least one part.  Both are refused before any launch."""
    import mla_latent_kv_40_b200 as mla
    dims = mla.make_dims(128, 512, 64, 128, 128, 7168, 64, "bf16", cache_layout=1)
    fake = ctypes.c_void_p(256)
    base = [ctypes.byref(dims), 4, 2, fake, fake, fake, fake, None, 2048, 8192, fake, 131072]
    tail = [fake, fake, fake, fake, 1 << 20, None, None]
    assert mla._lib.mla_decode_partial(*base, 32, 4096, *tail) == -1        # kv_begin not a multiple of 64
    assert mla._lib.mla_decode_partial(*base, 4096, 4096, *tail) == -1      # empty range
    tail_no_lse = [fake, fake, None, fake, 1 << 20, None, None]
    assert mla._lib.mla_decode_partial(*base, 0, 4096, *tail_no_lse) == -1  # lse is required
    n = ctypes.c_size_t(0)
    assert mla._lib.mla_merge_workspace_size(ctypes.byref(dims), 4, 2, 0, ctypes.byref(n)) == -1
    assert mla._lib.mla_merge_workspace_size(ctypes.byref(dims), 4, 2, 4, ctypes.byref(n)) == 0
    assert n.value >= 4 * 4 * 2 * 128 * 512 * 4
    # mla_merge_partials refuses missing parts and a short or misaligned workspace before any launch.
    merge = mla._lib.mla_merge_partials
    ws = ctypes.c_void_p(1 << 20)
    assert merge(ctypes.byref(dims), 4, 2, 4, None, fake, fake, fake, None, ws, n.value, None) == -1
    assert merge(ctypes.byref(dims), 4, 2, 4, fake, None, fake, fake, None, ws, n.value, None) == -1
    assert merge(ctypes.byref(dims), 4, 2, 4, fake, fake, fake, None, None, ws, n.value, None) == -1
    assert merge(ctypes.byref(dims), 4, 2, 4, fake, fake, fake, fake, None, ws, n.value - 256, None) == -3
    assert merge(ctypes.byref(dims), 4, 2, 4, fake, fake, fake, fake, None, ctypes.c_void_p((1 << 20) + 16), n.value,
                 None) == -3
    assert merge(ctypes.byref(dims), 4, 2, 0, fake, fake, fake, fake, None, ws, n.value, None) == -1
