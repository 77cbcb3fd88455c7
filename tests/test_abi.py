"""The C ABI library loads and exports what include/mla_decode.h declares (no GPU).

Only host-side paths run here: status strings, sizes, and argument checks that
return before any CUDA call.
"""
import ctypes
import os
import re
import subprocess

import pytest

from mla_paged_latent_decode_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla_decode.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    assert declared_functions() == sorted(binding.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(binding.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(mla_[a-z0-9_]+)$", out, flags=re.M))
    assert set(declared_functions()) <= exported


def test_library_links_no_cuda_driver_or_torch():
    out = subprocess.run(["readelf", "-d", binding.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    needed = re.findall(r"\(NEEDED\)\s+Shared library: \[(.+?)\]", out)
    assert not any(n.startswith("libcuda.so") for n in needed)
    assert not any("torch" in n for n in needed)


def test_error_strings():
    for code in range(8):
        assert binding.error_string(code).startswith("MLA_")
    assert "unknown" in binding.error_string(99)
    assert "sm_100a" in binding.version()


def test_workspace_size():
    ws = binding.workspace_size(64, 1, 128, 74)
    slots, rows = 64 + 74, 128
    expect = -(-(slots * rows * 512 * 4) // 256) * 256 + -(-(slots * rows * 4) // 256) * 256
    assert ws == expect
    assert binding.lib.mla_workspace_size(0, 1, 128, 512, 74) == 0
    assert binding.lib.mla_workspace_size(4, 1, 128, 256, 74) == 0


def _decode_raw(**kw):
    args = dict(q=1 << 12, kcache=1 << 12, num_blocks=4, block_table=1 << 12, bt_stride=3,
                cache_seqlens=1 << 12, batch=2, s_q=1, h_q=16, d=576, dv=512, scale=0.07,
                causal=0, tile_md=1 << 12, num_splits=1 << 12, num_workers=148,
                workspace=1 << 12, workspace_bytes=1 << 30, out=1 << 12, lse=1 << 12)
    args.update(kw)
    v = ctypes.c_void_p
    return binding.lib.mla_decode_kvcache(
        v(args["q"]), v(args["kcache"]), args["num_blocks"], v(args["block_table"]),
        args["bt_stride"], v(args["cache_seqlens"]), args["batch"], args["s_q"], args["h_q"],
        args["d"], args["dv"], args["scale"], args["causal"], v(args["tile_md"]),
        v(args["num_splits"]), args["num_workers"], v(args["workspace"]),
        args["workspace_bytes"], v(args["out"]), v(args["lse"]), v(0), v(0))


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), binding.MLA_ERR_INVALID_ARG),
    (dict(out=0), binding.MLA_ERR_INVALID_ARG),
    (dict(d=512), binding.MLA_ERR_UNSUPPORTED),
    (dict(dv=576), binding.MLA_ERR_UNSUPPORTED),
    (dict(batch=0), binding.MLA_ERR_INVALID_ARG),
    (dict(causal=2), binding.MLA_ERR_INVALID_ARG),
    (dict(num_workers=0), binding.MLA_ERR_INVALID_ARG),
    (dict(num_blocks=0), binding.MLA_ERR_INVALID_ARG),
    (dict(num_blocks=1 << 25), binding.MLA_ERR_INVALID_ARG),
    (dict(q=(1 << 12) + 2), binding.MLA_ERR_INVALID_ARG),
    (dict(workspace=(1 << 12) + 16), binding.MLA_ERR_INVALID_ARG),
    (dict(workspace_bytes=100), binding.MLA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), binding.MLA_ERR_INVALID_ARG),
    (dict(s_q=512, h_q=256), binding.MLA_ERR_UNSUPPORTED),
])
def test_decode_host_validation(kw, code):
    # every case fails validation before any CUDA call, so no device is needed
    assert _decode_raw(**kw) == code


def test_metadata_host_validation():
    v = ctypes.c_void_p
    assert binding.lib.mla_get_metadata(v(0), 2, 16, 1, v(4096), v(4096), 148, v(0)) == 1
    assert binding.lib.mla_get_metadata(v(4096), 0, 16, 1, v(4096), v(4096), 148, v(0)) == 1
    assert binding.lib.mla_get_metadata(v(4096), 2, 16, 1, v(4096), v(4096), 0, v(0)) == 1
    nw, st = ctypes.c_int(0), ctypes.c_int(0)
    assert binding.lib.mla_metadata_shape(0, 16, 1, ctypes.byref(nw), ctypes.byref(st)) == 1


def _append_raw(**kw):
    args = dict(rows=1 << 12, s_new=1, kcache=1 << 12, num_blocks=4, block_table=1 << 12,
                bt_stride=3, seqlens=1 << 12, batch=2, free_pages=1 << 12, free_capacity=4,
                free_count=1 << 12)
    args.update(kw)
    v = ctypes.c_void_p
    return binding.lib.mla_append_latent(
        v(args["rows"]), args["s_new"], v(args["kcache"]), args["num_blocks"],
        v(args["block_table"]), args["bt_stride"], v(args["seqlens"]), args["batch"],
        v(args["free_pages"]), args["free_capacity"], v(args["free_count"]), v(0), v(0))


@pytest.mark.parametrize("kw", [dict(rows=0), dict(kcache=0), dict(block_table=0),
                                dict(seqlens=0), dict(free_pages=0), dict(free_count=0),
                                dict(s_new=0), dict(s_new=65537), dict(batch=0),
                                dict(batch=65537), dict(bt_stride=0), dict(free_capacity=0),
                                dict(num_blocks=0), dict(num_blocks=1 << 25),
                                dict(rows=(1 << 12) + 8), dict(kcache=(1 << 12) + 4)])
def test_append_host_validation(kw):
    assert _append_raw(**kw) == binding.MLA_ERR_INVALID_ARG


def test_release_host_validation():
    v = ctypes.c_void_p
    ok = dict(mask=1 << 12, bt=1 << 12, stride=3, sl=1 << 12, batch=2, fp=1 << 12, cap=4, fc=1 << 12)

    def call(**kw):
        a = dict(ok, **kw)
        return binding.lib.mla_release_pages(v(a["mask"]), v(a["bt"]), a["stride"], v(a["sl"]),
                                             a["batch"], v(a["fp"]), a["cap"], v(a["fc"]), v(0),
                                             v(0))
    for kw in (dict(mask=0), dict(bt=0), dict(sl=0), dict(fp=0), dict(fc=0), dict(stride=0),
               dict(batch=0), dict(cap=0)):
        assert call(**kw) == binding.MLA_ERR_INVALID_ARG


def _fp8_decode_raw(**kw):
    args = dict(q=1 << 12, kcache=1 << 12, kscale=1 << 12, num_blocks=4, block_table=1 << 12,
                bt_stride=3, cache_seqlens=1 << 12, batch=2, s_q=1, h_q=16, d=576, dv=512,
                scale=0.07, causal=0, tile_md=1 << 12, num_splits=1 << 12, num_workers=148,
                workspace=1 << 12, workspace_bytes=1 << 30, out=1 << 12, lse=1 << 12)
    args.update(kw)
    v = ctypes.c_void_p
    return binding.lib.mla_decode_kvcache_fp8(
        v(args["q"]), v(args["kcache"]), v(args["kscale"]), args["num_blocks"],
        v(args["block_table"]), args["bt_stride"], v(args["cache_seqlens"]), args["batch"],
        args["s_q"], args["h_q"], args["d"], args["dv"], args["scale"], args["causal"],
        v(args["tile_md"]), v(args["num_splits"]), args["num_workers"], v(args["workspace"]),
        args["workspace_bytes"], v(args["out"]), v(args["lse"]), v(0), v(0))


@pytest.mark.parametrize("kw,code", [
    (dict(kscale=0), binding.MLA_ERR_INVALID_ARG),
    (dict(kcache=0), binding.MLA_ERR_INVALID_ARG),
    (dict(kscale=(1 << 12) + 4), binding.MLA_ERR_INVALID_ARG),
    (dict(s_q=2, h_q=65536), binding.MLA_ERR_UNSUPPORTED),   # more than 65536 query rows
    (dict(d=512), binding.MLA_ERR_UNSUPPORTED),
    (dict(causal=3), binding.MLA_ERR_INVALID_ARG),
    (dict(workspace_bytes=64), binding.MLA_ERR_INVALID_ARG),
])
def test_fp8_decode_host_validation(kw, code):
    assert _fp8_decode_raw(**kw) == code


def test_fp8_append_host_validation():
    v = ctypes.c_void_p
    ok = dict(rows=1 << 12, s_new=1, kc=1 << 12, ks=1 << 12, nb=4, bt=1 << 12, stride=3,
              sl=1 << 12, batch=2, fp=1 << 12, cap=4, fc=1 << 12)

    def call(**kw):
        a = dict(ok, **kw)
        return binding.lib.mla_append_latent_fp8(
            v(a["rows"]), a["s_new"], v(a["kc"]), v(a["ks"]), a["nb"], v(a["bt"]), a["stride"],
            v(a["sl"]), a["batch"], v(a["fp"]), a["cap"], v(a["fc"]), v(0), v(0))
    for kw in (dict(ks=0), dict(kc=0), dict(rows=0), dict(ks=(1 << 12) + 8), dict(s_new=0),
               dict(batch=0), dict(nb=1 << 25)):
        assert call(**kw) == binding.MLA_ERR_INVALID_ARG, kw


def test_sparse_workspace_size_and_validation():
    lib = binding.lib
    pos, topk, h_q, W = 2 * 3, 100, 16, 148
    r = lambda n: -(-n // 256) * 256
    dec = binding.workspace_size(pos, 1, h_q, W)
    # cached rows of the used entries, counts, metadata, lse per position, decode partials
    # (the decode copies the selected rows itself: no gathered pages)
    expect = (r(pos * topk * 4) + r(pos * 4) + r(W * 8 * 4) + r((pos + 1) * 4)
              + r(pos * h_q * 4) + dec)
    assert lib.mla_sparse_workspace_size(2, 3, h_q, topk, W) == expect
    assert lib.mla_sparse_workspace_size(2, 3, h_q, 0, W) == 0
    v = ctypes.c_void_p
    ok = dict(q=1 << 12, kc=1 << 12, nb=4, bt=1 << 12, stride=3, sl=1 << 12, batch=2, s_q=3,
              h_q=16, d=576, dv=512, idx=1 << 12, topk=100, scale=0.07, causal=0, W=148,
              ws=1 << 12, wsb=1 << 40, out=1 << 12, lse=1 << 12)

    def call(**kw):
        a = dict(ok, **kw)
        return lib.mla_decode_sparse(
            v(a["q"]), v(a["kc"]), a["nb"], v(a["bt"]), a["stride"], v(a["sl"]), a["batch"],
            a["s_q"], a["h_q"], a["d"], a["dv"], v(a["idx"]), a["topk"], a["scale"], a["causal"],
            a["W"], v(a["ws"]), a["wsb"], v(a["out"]), v(a["lse"]), v(0), v(0))
    for kw, code in ((dict(idx=0), binding.MLA_ERR_INVALID_ARG),
                     (dict(topk=0), binding.MLA_ERR_INVALID_ARG),
                     (dict(topk=65537), binding.MLA_ERR_INVALID_ARG),
                     (dict(d=512), binding.MLA_ERR_UNSUPPORTED),
                     (dict(ws=(1 << 12) + 16), binding.MLA_ERR_INVALID_ARG),
                     (dict(wsb=1000), binding.MLA_ERR_INVALID_ARG),
                     (dict(batch=70000), binding.MLA_ERR_INVALID_ARG),
                     (dict(scale=float("inf")), binding.MLA_ERR_INVALID_ARG)):
        assert call(**kw) == code, kw


def test_binding_rejects_bad_tensors_before_any_call():
    # checks that stay on under `python -O`: CPU tensors and wrong dtypes raise ValueError
    import torch
    with pytest.raises(ValueError):
        binding.get_mla_metadata(torch.zeros(3, dtype=torch.int32), 16, 1)
    with pytest.raises(ValueError):
        binding.get_mla_metadata(torch.zeros(3, dtype=torch.int64), 16, 1)
    q = torch.zeros((1, 1, 16, 576), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        binding.mla_decode_sparse(q, torch.zeros((1, 64, 576), dtype=torch.bfloat16),
                                  torch.zeros((1, 1), dtype=torch.int32),
                                  torch.ones(1, dtype=torch.int32),
                                  torch.zeros((1, 1, 4), dtype=torch.int32), 0.07)


def _decode_args(b=2, s_q=1, h_q=16, nb=4, W=8):
    import torch
    return dict(
        q=torch.zeros((b, s_q, h_q, 576), dtype=torch.bfloat16),
        kcache=torch.zeros((nb, 64, 576), dtype=torch.bfloat16),
        block_table=torch.zeros((b, 3), dtype=torch.int32),
        cache_seqlens=torch.ones(b, dtype=torch.int32),
        dv=512,
        tile_md=torch.zeros((W, 8), dtype=torch.int32),
        num_splits=torch.zeros(b + 1, dtype=torch.int32),
        softmax_scale=0.07,
        out=torch.zeros((b, s_q, h_q, 512), dtype=torch.bfloat16),
        lse=torch.zeros((b, h_q, s_q), dtype=torch.float32),
        workspace=torch.zeros(1 << 20, dtype=torch.uint8),
        device_status=torch.zeros(1, dtype=torch.int32))


@pytest.mark.parametrize("field,bad,match", [
    ("cache_seqlens", "short", "cache_seqlens must have shape"),
    ("cache_seqlens", "int64", "cache_seqlens must be torch.int32"),
    ("num_splits", "short", "num_splits must have shape"),
    ("tile_md", "stride", r"tile_md must be \[num_workers, 8\]"),
    ("tile_md", "int64", "tile_md must be torch.int32"),
    ("out", "short", "out must have shape"),
    ("out", "fp32", "out must be torch.bfloat16"),
    ("lse", "transposed", "lse must have shape"),
    ("lse", "fp16", "lse must be torch.float32"),
    ("workspace", "fp32", "workspace must be a contiguous 1-D uint8"),
    ("device_status", "int64", "device_status must hold one int32"),
    ("block_table", "rows", r"block_table must be \[batch, max_pages\]"),
    ("kcache", "page", r"kcache must be \[num_blocks, 64, 576\]"),
    ("q", "dims", r"q must be \[batch, s_q, h_q, 576\]"),
])
def test_binding_checks_every_extent(field, bad, match):
    # each tensor whose extent the kernels rely on is checked before the call;
    # the C ABI itself sees only pointers
    import torch
    a = _decode_args()
    t = a[field]
    if bad == "short":
        t = t.flatten()[:-1] if t.dim() == 1 else t[:-1]
    elif bad == "int64":
        t = t.to(torch.int64)
    elif bad == "stride":
        t = torch.zeros((t.shape[0], 4), dtype=torch.int32)
    elif bad == "fp32":
        t = t.float()
    elif bad == "fp16":
        t = t.half()
    elif bad == "transposed":
        t = t.transpose(1, 2).contiguous()
    elif bad == "rows":
        t = torch.zeros((1, 3), dtype=torch.int32)
    elif bad == "page":
        t = torch.zeros((4, 32, 576), dtype=torch.bfloat16)
    elif bad == "dims":
        t = torch.zeros((2, 1, 16, 512), dtype=torch.bfloat16)
    a[field] = t
    with pytest.raises(ValueError, match=match):
        binding.mla_decode_kvcache(**a)


def test_binding_well_formed_cpu_tensors_stop_at_device_check():
    with pytest.raises(ValueError, match="CUDA device"):
        binding.mla_decode_kvcache(**_decode_args())


def test_static_scratch_checks_arguments_before_the_limit():
    # a shape whose workspace exceeds the static array, but with a null pointer:
    # the argument error is reported, not the limit
    lib = binding.lib
    b, s_q, h_q, nw = 1024, 1, 128, 74
    assert binding.workspace_size(b, s_q, h_q, nw) > binding.STATIC_SCRATCH_BYTES
    v = ctypes.c_void_p

    def call(q=1 << 12, lse=1 << 12, d=576, batch=b):
        return lib.mla_decode_kvcache_static_scratch(
            v(q), v(1 << 12), 1, v(1 << 12), 1, v(1 << 12), batch, s_q, h_q, d, 512, 0.07, 0,
            v(1 << 12), v(1 << 12), nw, v(1 << 12), v(lse), v(0), v(0))
    assert call(q=0) == binding.MLA_ERR_INVALID_ARG
    assert call(lse=0) == binding.MLA_ERR_INVALID_ARG
    assert call(d=512) == binding.MLA_ERR_UNSUPPORTED
    assert call(batch=0) == binding.MLA_ERR_INVALID_ARG
    # well-formed arguments: the limit is reported, before any device call
    assert call() == binding.MLA_ERR_SCRATCH_LIMIT


def test_wait_limit_setting_is_clamped():
    # the device wait limit (a host-side setting read at each decode launch)
    assert binding.set_wait_limit_ns(5) == 2_000_000_000
    assert binding.set_wait_limit_ns(10**12) == 1000       # 5 ns was raised to 1 us
    assert binding.set_wait_limit_ns(0) == 2_000_000_000   # 10^12 was lowered to 2 s
    assert binding.set_wait_limit_ns(0) == 2_000_000_000


def test_merge_host_validation():
    lib = binding.lib
    v = ctypes.c_void_p
    ok = dict(outs=1 << 12, lses=1 << 12, R=2, b=2, s_q=1, h_q=16, out=1 << 13, lse=1 << 13)

    def call(**kw):
        a = dict(ok, **kw)
        return lib.mla_merge_partials(v(a["outs"]), v(a["lses"]), a["R"], a["b"], a["s_q"],
                                      a["h_q"], v(a["out"]), v(a["lse"]), v(0))
    for kw in (dict(outs=0), dict(lses=0), dict(out=0), dict(lse=0), dict(R=0), dict(R=4097),
               dict(b=0), dict(s_q=0), dict(h_q=0), dict(outs=(1 << 12) + 8),
               dict(out=(1 << 13) + 8), dict(lse=(1 << 13) + 2), dict(s_q=512, h_q=256),
               dict(R=4096, b=1 << 16, h_q=128)):
        assert call(**kw) == binding.MLA_ERR_INVALID_ARG, kw


@pytest.mark.parametrize("bad,match", [
    ("rows_fp32", "rows must be contiguous bf16"),
    ("codes_bf16", "kcache8 must be contiguous uint8"),
    ("codes_page", r"kcache8 must be \[num_blocks, 64, 576\]"),
    ("scale_fp16", "kscale must be contiguous fp32"),
    ("scale_device", "kscale must be contiguous fp32 on the rows' device"),
    ("scale_short", r"kscale must be \[num_blocks, 64\]"),
])
def test_fp8_append_checks_codes_and_scales(bad, match):
    # the FP8 append writes codes and scales through raw pointers: every extent,
    # type and device is checked before the call
    import torch
    b, nb = 2, 4
    rows = torch.zeros((b, 3, 576), dtype=torch.bfloat16)
    codes = torch.zeros((nb, 64, 576), dtype=torch.uint8)
    scales = torch.ones((nb, 64), dtype=torch.float32)
    if bad == "rows_fp32":
        rows = rows.float()
    elif bad == "codes_bf16":
        codes = codes.to(torch.bfloat16)
    elif bad == "codes_page":
        codes = torch.zeros((nb, 32, 576), dtype=torch.uint8)
    elif bad == "scale_fp16":
        scales = scales.half()
    elif bad == "scale_device":
        scales = torch.ones((nb, 64), dtype=torch.float32, device="meta")
    elif bad == "scale_short":
        scales = scales[:, :32].contiguous()
    with pytest.raises(ValueError, match=match):
        binding.append_latent_fp8(rows, codes, scales,
                                  torch.zeros((b, 3), dtype=torch.int32),
                                  torch.zeros(b, dtype=torch.int32),
                                  torch.arange(nb, dtype=torch.int32),
                                  torch.tensor([nb], dtype=torch.int32))


def test_missing_library_fails_loudly(tmp_path):
    # no fallback: without the built library the binding refuses to import
    import sys
    env = dict(os.environ, MLA_DECODE_LIB=str(tmp_path / "absent.so"))
    r = subprocess.run([sys.executable, "-c", "import mla_paged_latent_decode_b200.binding"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "not built" in r.stderr


def test_product_code_never_reaches_the_oracle():
    # the package and the C ABI neither import nor link anything under oracle/
    pkg = os.path.join(ROOT, "mla_paged_latent_decode_b200")
    pat = re.compile(r"^\s*(import\s+oracle|from\s+oracle\b|#include\s+[<\"].*oracle)", re.M)
    for dirpath, _, files in os.walk(pkg):
        for name in files:
            if name.endswith((".py", ".cu", ".cuh", ".h")):
                with open(os.path.join(dirpath, name)) as f:
                    assert not pat.search(f.read()), name
    for name in os.listdir(os.path.join(ROOT, "include")):
        with open(os.path.join(ROOT, "include", name)) as f:
            assert not pat.search(f.read()), name
