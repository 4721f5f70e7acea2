"""The C ABI library: it builds for sm_100a, loads, exports every declared symbol, and rejects bad
arguments before touching the GPU (CPU only: no call here launches a kernel)."""
import ctypes
import os
import re

import pytest

import periodic_sparse_attention_b200 as pia
from periodic_sparse_attention_b200 import build as pbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(pi_attn_\w+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    pbuild.build()
    return pia.load()


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ["pi_attn_fwd", "pi_attn_decode", "pi_attn_debug_index_sets", "pi_attn_check",
                 "pi_attn_status_string"]:
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
        assert name in pia.SIGNATURES, f"{name} has no Python binding"


def test_status_strings_and_version(lib):
    assert lib.pi_attn_status_string(0) == b"PI_ATTN_OK"
    assert lib.pi_attn_status_string(4) == b"PI_ATTN_EDEVICE"
    assert lib.pi_attn_version() >= 100


FAKE = ctypes.c_void_p(0x10000)  # aligned, never dereferenced: every call below fails validation first


def _fwd(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, w=FAKE, b=FAKE, out=FAKE, lse=None, B=1, H=1, n=16, d=64, kw=4, pi=4, S=2,
             dt=pia.PI_ATTN_BF16, path=0)
    a.update(kw)
    return lib.pi_attn_fwd_ex(a["q"], a["k"], a["v"], a["w"], a["b"], a["out"], a["lse"], a["B"], a["H"], a["n"],
                              a["d"], a["kw"], a["pi"], a["S"], a["dt"], a["path"], None)


@pytest.mark.parametrize("bad", [
    dict(q=None), dict(out=None), dict(w=None), dict(B=0), dict(H=0), dict(n=0), dict(d=0), dict(d=300),
    dict(d=12), dict(kw=-1), dict(pi=0), dict(S=-1), dict(dt=7), dict(path=9), dict(q=ctypes.c_void_p(0x10008)),
    dict(dt=pia.PI_ATTN_F32, d=6),
])
def test_fwd_rejects_bad_arguments(lib, bad):
    assert _fwd(lib, **bad) == pia.PI_ATTN_EINVAL
    assert lib.pi_attn_last_error() != b""


def test_tensor_core_path_is_explicit_about_coverage(lib):
    assert _fwd(lib, dt=pia.PI_ATTN_F32, d=32, path=pia.PATHS["tc"]) in (pia.PI_ATTN_EUNSUPPORTED,)
    assert _fwd(lib, d=96, path=pia.PATHS["tc"]) == pia.PI_ATTN_EUNSUPPORTED


def test_decode_and_index_export_reject_bad_arguments(lib):
    assert lib.pi_attn_decode(FAKE, FAKE, None, FAKE, FAKE, None, FAKE, None, 1, 1, 8, 64, 4, 4, 2, 1, None) == \
        pia.PI_ATTN_EINVAL
    assert lib.pi_attn_decode(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, None, 1, 1, 0, 64, 4, 4, 2, 1, None) == \
        pia.PI_ATTN_EINVAL
    assert lib.pi_attn_debug_index_sets(16, 4, 4, 2, FAKE, FAKE, 3, None) == pia.PI_ATTN_EINVAL  # width too small
    assert lib.pi_attn_debug_index_sets(16, 4, 0, 2, FAKE, FAKE, 16, None) == pia.PI_ATTN_EINVAL


def test_plan_reports_launches_and_scratch(lib):
    assert pia.pi_attn_fwd_plan(1, 8, 4096, 64, 128, 64, 4, "bf16", "tc_fused") == (1, 0)
    assert pia.pi_attn_fwd_plan(1, 8, 4096, 64, 128, 64, 4, "bf16", "tc_split") == (2, 8 * 4096 * (2 * 64 + 4))
    assert pia.pi_attn_fwd_plan(1, 32, 131072, 128, 512, 1024, 16, "bf16", "auto")[0] == 2
    assert pia.pi_attn_fwd_plan(1, 2, 256, 32, 8, 16, 2, "f32", "auto") == (1, 0)
    # n % pi != 0: the residue view covers rows [0, 62 * 64); the tiles from row 3968 on (tile 31,
    # which reaches past the whole periods) run the single pass -- three launches
    assert pia.pi_attn_fwd_plan(1, 8, 4000, 64, 128, 64, 4, "bf16", "tc_split")[0] == 3
    # n % pi != 0 with the whole periods ending on a tile boundary: 2 * 128 rows, then a tail
    assert pia.pi_attn_fwd_plan(1, 1, 300, 64, 10, 128, 3, "bf16", "tc_split")[0] == 3
    # fewer rows than one period: no residue view
    with pytest.raises(pia.PiAttnError):
        pia.pi_attn_fwd_plan(1, 8, 100, 64, 16, 128, 4, "bf16", "tc_split")


def test_workspace_is_checked_before_any_launch(lib):
    # split path (n % pi == 0, skips outside the window): B*H*n*(2d+4) bytes of workspace
    need = 2 * 4096 * (2 * 64 + 4)
    args = [FAKE] * 7 + [1, 2, 4096, 64, 128, 64, 4, pia.PI_ATTN_BF16, pia.PATHS["tc_split"]]
    assert lib.pi_attn_fwd_ws(*args, ctypes.c_void_p(0x10008), need, None) == pia.PI_ATTN_EINVAL  # misaligned
    assert b"aligned" in lib.pi_attn_last_error()
    assert lib.pi_attn_fwd_ws(*args, FAKE, need - 1, None) == pia.PI_ATTN_EINVAL  # one byte short
    assert str(need).encode() in lib.pi_attn_last_error()
    assert pia.pi_attn_fwd_plan(1, 2, 4096, 64, 128, 64, 4, "bf16", "tc_split") == (2, need)


def test_bidir_split_is_refused_before_any_launch(lib):
    # the bidirectional split needs whole periods (a forward skip may reach past the last one)
    args = [FAKE] * 7 + [1, 1, 4000, 64, 128, 64, 4, pia.PI_ATTN_BF16, pia.PATHS["tc_split"], None]
    assert lib.pi_attn_fwd_bidir(*args) == pia.PI_ATTN_EUNSUPPORTED
    assert b"n % pi == 0" in lib.pi_attn_last_error()
    assert lib.pi_attn_debug_index_sets_bidir(16, 4, 4, 2, FAKE, FAKE, 4 + 1 + 2, None) == pia.PI_ATTN_EINVAL  # < 2k+1+2S


def test_backward_rejects_bad_arguments(lib):
    g = [FAKE] * 5
    # every call below is refused by the argument checks before anything is launched
    base = [FAKE] * 6 + g + [1, 2, 64, 64, 8, 16, 2, pia.PI_ATTN_BF16, 0, None, 0, None]
    bad = list(base)
    bad[6] = None  # dq
    assert lib.pi_attn_bwd(*bad) == pia.PI_ATTN_EINVAL
    bad = list(base)
    bad[7] = ctypes.c_void_p(0x10008)  # dk misaligned
    assert lib.pi_attn_bwd(*bad) == pia.PI_ATTN_EINVAL
    bad = list(base)
    bad[-3] = FAKE  # a workspace that is too small
    bad[-2] = 16
    assert lib.pi_attn_bwd(*bad) == pia.PI_ATTN_EINVAL
    assert lib.pi_attn_bwd_workspace_bytes(1, 2, 64, 64) == 4 * (5 * 2 * 64 + 2 * 2 * 65)


def test_ring_cache_arguments_are_checked_before_any_launch(lib):
    # capacity below max(k_win, S*pi) + 1 = 81
    assert lib.pi_attn_decode_ring(*([FAKE] * 8), 1, 1, 80, 64, 40, 16, 5, pia.PI_ATTN_BF16, None) == pia.PI_ATTN_EINVAL
    # no cache_len
    args = [FAKE] * 5 + [None] + [FAKE] * 2
    assert lib.pi_attn_decode_ring(*args, 1, 1, 81, 64, 40, 16, 5, pia.PI_ATTN_BF16, None) == pia.PI_ATTN_EINVAL
    # fp32 is not covered
    assert lib.pi_attn_decode_ring(*([FAKE] * 8), 1, 1, 81, 64, 40, 16, 5, pia.PI_ATTN_F32, None) == \
        pia.PI_ATTN_EUNSUPPORTED
    assert lib.pi_attn_cache_append(FAKE, FAKE, FAKE, FAKE, None, 1, 1, 81, 64, pia.PI_ATTN_BF16, 1, None) == \
        pia.PI_ATTN_EINVAL


def test_shard_arguments_are_checked_before_any_launch(lib):
    # B H n_q n_kv row0 kv0 d k_win pi S; reach = max(40, 5 * 16) = 80
    def call(n_q, n_kv, row0, kv0, d=64, dtype=pia.PI_ATTN_BF16):
        return lib.pi_attn_fwd_shard(*([FAKE] * 7), 1, 2, n_q, n_kv, row0, kv0, d, 40, 16, 5, dtype, None)
    # every call below fails its checks, so none launches (the pointers are placeholders)
    assert call(100, 179, 200, 121) == pia.PI_ATTN_EINVAL   # halo starts at 121, after row 200 - 80
    assert call(100, 179, 200, 120) == pia.PI_ATTN_EINVAL   # k/v rows end at 298, before row 299
    assert call(100, 150, 200, 100) == pia.PI_ATTN_EINVAL   # ... and here at 249
    assert call(0, 180, 200, 120) == pia.PI_ATTN_EINVAL     # empty shard
    assert call(100, 180, -1, 0) == pia.PI_ATTN_EINVAL      # negative row
    assert call(100, 180, 200, 120, dtype=pia.PI_ATTN_F32) == pia.PI_ATTN_EUNSUPPORTED
    assert call(100, 180, 200, 120, d=32) == pia.PI_ATTN_EUNSUPPORTED


def test_tensor_core_backward_arguments_are_checked_before_any_launch(lib):
    args = [FAKE] * 11
    # fp32 and d = 32 are not covered by the tensor-core path; an unknown path is refused
    assert lib.pi_attn_bwd_ex(*args, 1, 2, 64, 64, 8, 16, 2, pia.PI_ATTN_F32, 0, 2, None, 0, None) == \
        pia.PI_ATTN_EUNSUPPORTED
    assert lib.pi_attn_bwd_ex(*args, 1, 2, 64, 32, 8, 16, 2, pia.PI_ATTN_BF16, 0, 2, None, 0, None) == \
        pia.PI_ATTN_EUNSUPPORTED
    assert lib.pi_attn_bwd_ex(*args, 1, 2, 64, 64, 8, 16, 2, pia.PI_ATTN_BF16, 0, 7, None, 0, None) == \
        pia.PI_ATTN_EINVAL
    # a workspace smaller than the path needs
    tc = lib.pi_attn_bwd_workspace_bytes_ex(1, 2, 64, 64, pia.PI_ATTN_BF16, 2)
    simt = lib.pi_attn_bwd_workspace_bytes_ex(1, 2, 64, 64, pia.PI_ATTN_BF16, 1)
    rows = 1 * 2 * 64
    # the rows' five terms and the gate partials, then the forward's out (bf16) and lse
    assert simt == lib.pi_attn_bwd_workspace_bytes(1, 2, 64, 64) and tc >= 4 * 5 * rows + rows * (2 * 64 + 4)
    assert lib.pi_attn_bwd_ex(*args, 1, 2, 64, 64, 8, 16, 2, pia.PI_ATTN_BF16, 0, 2, FAKE, tc - 16, None) == \
        pia.PI_ATTN_EINVAL
    # the fused and split tensor-core paths take the same workspace (the split's skip partials
    # live in dq until the dq passes write it)
    assert lib.pi_attn_bwd_workspace_bytes_ex(1, 2, 64, 64, pia.PI_ATTN_BF16, 3) == tc
    assert lib.pi_attn_bwd_workspace_bytes_ex(1, 2, 64, 64, pia.PI_ATTN_BF16, 4) == tc
    split = pia.BWD_PATHS["tc_split"]
    assert lib.pi_attn_bwd_ex(*args, 1, 2, 64, 64, 8, 16, 2, pia.PI_ATTN_BF16, 1, split, None, 0, None) == \
        pia.PI_ATTN_EUNSUPPORTED  # bidirectional
    assert lib.pi_attn_bwd_ex(*args, 1, 2, 60, 64, 8, 16, 2, pia.PI_ATTN_BF16, 0, split, None, 0, None) == \
        pia.PI_ATTN_EUNSUPPORTED  # n not a whole number of periods
    assert lib.pi_attn_bwd_ex(*args, 1, 2, 64, 64, 40, 16, 2, pia.PI_ATTN_BF16, 0, split, None, 0, None) == \
        pia.PI_ATTN_EUNSUPPORTED  # no skip outside the window (m0 = 3 > S)
    assert lib.pi_attn_bwd_ex(*args, 1, 2, 64, 64, 8, 16, 2, pia.PI_ATTN_BF16, 0, 5, None, 0, None) == \
        pia.PI_ATTN_EINVAL


def test_built_for_sm100a_only():
    cmd = pbuild.command("x.so")
    assert "arch=compute_100a,code=sm_100a" in cmd and "-lineinfo" in cmd


def test_product_path_never_touches_the_oracle():
    pkg = os.path.join(ROOT, "periodic_sparse_attention_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in text and "from oracle" not in text and "pi_oracle" not in text, fn


def test_binding_fails_loudly_without_the_library(tmp_path):
    with pytest.raises(ImportError):
        pia.load(str(tmp_path / "missing.so"))


def test_host_entry_workspace_size_and_argument_checks(lib):
    # three rotating chunk buffers (q, k, v, out and lse of chunk_heads heads, 256-byte rounded)
    # and the split path's scratch for one chunk
    r = lambda x: (x + 255) // 256 * 256  # noqa: E731
    B, H, n, d = 1, 32, 131072, 128
    for chunk, hc in ((4, 4), (0, 1), (100, 32), (1, 1)):
        want = 3 * (4 * r(hc * n * d * 2) + r(hc * n * 4)) + r(hc * n * (2 * d + 4))
        assert lib.pi_attn_fwd_host_workspace_bytes(B, H, n, d, pia.PI_ATTN_BF16, chunk) == want
    assert lib.pi_attn_fwd_host_workspace_bytes(1, 5, 300, 32, pia.PI_ATTN_F32, 0) == \
        3 * (4 * r(300 * 32 * 4) + r(300 * 4)) + r(300 * 68)
    for bad in ((0, 1, 1, 64, 1, 0), (1, 1, 1, 64, 1, -1), (1, 1, 1, 64, 7, 0)):
        assert lib.pi_attn_fwd_host_workspace_bytes(*bad) == -1
    # rejected before any CUDA call: no device is needed for these
    h = ctypes.c_void_p(0x1000)  # stand-in pointers, never dereferenced
    ws = ctypes.c_void_p(0x10000)
    need = lib.pi_attn_fwd_host_workspace_bytes(1, 2, 256, 64, pia.PI_ATTN_BF16, 1)

    def call(q=h, wg=h, chunk=1, w=ws, nbytes=need, n=256, pi=16, path=0):
        return lib.pi_attn_fwd_host(q, h, h, wg, h, h, None, 1, 2, n, 64, 16, pi, 3, pia.PI_ATTN_BF16, path, chunk, w,
                                    nbytes, None)
    assert call(q=None) == pia.PI_ATTN_EINVAL
    assert call(wg=None) == pia.PI_ATTN_EINVAL
    assert call(chunk=-1) == pia.PI_ATTN_EINVAL
    assert call(w=None) == pia.PI_ATTN_EINVAL
    assert call(w=ctypes.c_void_p(0x10010)) == pia.PI_ATTN_EINVAL  # not 256-byte aligned
    assert call(nbytes=need - 1) == pia.PI_ATTN_EINVAL
    assert call(pi=0) == pia.PI_ATTN_EINVAL
    assert call(n=100, path=pia.PATHS["tc_split"], pi=128) == pia.PI_ATTN_EUNSUPPORTED  # n < pi


def test_tensor_core_paths_refuse_more_than_65535_heads_before_any_launch(lib):
    # the tensor-core grids take (b, h) as their y dimension: an explicit tensor-core path refuses
    # B*H > 65535 up front; the automatic choice takes the CUDA-core kernel (the plan shows it)
    args = [FAKE] * 7 + [2, 40000, 256, 64, 16, 32, 2, pia.PI_ATTN_BF16]
    for path in ("tc", "tc_fused", "tc_split"):
        assert lib.pi_attn_fwd_ex(*args, pia.PATHS[path], None) == pia.PI_ATTN_EUNSUPPORTED
        assert b"65535" in lib.pi_attn_last_error()
    assert pia.pi_attn_fwd_plan(2, 40000, 256, 64, 16, 32, 2, "bf16", "auto") == (1, 0)
    assert lib.pi_attn_fwd_shard(*([FAKE] * 7), 2, 40000, 128, 256, 128, 0, 64, 16, 32, 2, pia.PI_ATTN_BF16,
                                 None) == pia.PI_ATTN_EUNSUPPORTED


def test_backward_host_entry_workspace_size_and_argument_checks(lib):
    r = lambda x: (x + 255) // 256 * 256  # noqa: E731
    B, H, n, d = 2, 16, 32768, 128
    for chunk, hc in ((0, 1), (4, 4), (64, 16)):
        per = B * hc * n * d
        want = 3 * (4 * r(per * 2) + 3 * r(per * 4)) + \
            r(lib.pi_attn_bwd_workspace_bytes_ex(B, hc, n, d, pia.PI_ATTN_BF16, pia.BWD_PATHS["tc"]))
        assert lib.pi_attn_bwd_host_workspace_bytes(B, H, n, d, pia.PI_ATTN_BF16, pia.BWD_PATHS["tc"], chunk) == want
    assert lib.pi_attn_bwd_host_workspace_bytes(1, 1, 1, 64, pia.PI_ATTN_BF16, 9, 0) == -1  # unknown path
    assert lib.pi_attn_bwd_host_workspace_bytes(1, 1, 1, 64, pia.PI_ATTN_BF16, 0, -2) == -1
    h = ctypes.c_void_p(0x1000)
    ws = ctypes.c_void_p(0x10000)
    need = lib.pi_attn_bwd_host_workspace_bytes(1, 2, 256, 64, pia.PI_ATTN_BF16, 0, 1)

    def call(q=h, dw=h, chunk=1, w=ws, nbytes=need, path=0, bidir=0, n=256, pi=16):
        return lib.pi_attn_bwd_host(q, h, h, h, h, h, h, h, h, dw, h, 1, 2, n, 64, 16, pi, 3, pia.PI_ATTN_BF16, bidir,
                                    path, chunk, w, nbytes, None)
    assert call(q=None) == pia.PI_ATTN_EINVAL
    assert call(dw=None) == pia.PI_ATTN_EINVAL
    assert call(chunk=-1) == pia.PI_ATTN_EINVAL
    assert call(w=ctypes.c_void_p(0x10010)) == pia.PI_ATTN_EINVAL
    assert call(nbytes=need - 1) == pia.PI_ATTN_EINVAL
    assert call(path=pia.BWD_PATHS["tc_split"], bidir=1) == pia.PI_ATTN_EUNSUPPORTED
    assert call(path=pia.BWD_PATHS["tc_split"], n=250) == pia.PI_ATTN_EUNSUPPORTED  # n % pi != 0


def test_shard_scratch_and_workspace_checks_before_any_launch(lib):
    # the split path's scratch where the shard's rows and halo start on whole periods; none otherwise
    B, H, d = 1, 32, 128
    assert lib.pi_attn_fwd_shard_scratch_bytes(B, H, 16384, 16384, 0, d, 512, 1024, 16) == B * H * 16384 * (2 * d + 4)
    assert lib.pi_attn_fwd_shard_scratch_bytes(B, H, 16384, 16000, 0, d, 512, 1024, 16) == 0     # row0 off a period
    assert lib.pi_attn_fwd_shard_scratch_bytes(B, H, 16384, 16384, 100, d, 512, 1024, 16) == 0   # halo off a period
    assert lib.pi_attn_fwd_shard_scratch_bytes(B, H, 4096, 0, 0, 64, 128, 64, 4) == 0            # single pass shape
    assert lib.pi_attn_fwd_shard_scratch_bytes(0, H, 16, 0, 0, d, 1, 1, 1) == -1
    need = lib.pi_attn_fwd_shard_scratch_bytes(1, 2, 2048, 2048, 0, 64, 128, 256, 16)
    assert need > 0
    args = [FAKE] * 7 + [1, 2, 2048, 4096, 2048, 0, 64, 128, 256, 16, pia.PI_ATTN_BF16]
    assert lib.pi_attn_fwd_shard_ws(*args, ctypes.c_void_p(0x10008), need, None) == pia.PI_ATTN_EINVAL  # misaligned
    assert lib.pi_attn_fwd_shard_ws(*args, FAKE, need - 1, None) == pia.PI_ATTN_EINVAL  # one byte short
