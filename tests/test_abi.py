"""The C-ABI library: it loads, exports every symbol include/fa.h declares, and its
host-side argument checks return the documented codes without touching a device.

Pointers below are fake integers; every case is rejected before any CUDA call, so these
tests run on a CPU-only machine (and launch nothing on a GPU machine)."""
import ctypes
import math
import subprocess

import pytest
import torch

from exact_io_aware_59_b200 import binding
from exact_io_aware_59_b200 import build as fa_build

A = 1 << 20  # fake, 16-byte aligned, non-overlapping "device" addresses
Q, K, V, O, L = A * 1, A * 2, A * 3, A * 4, A * 5


def _fwd(**kw):
    args = dict(q=Q, k=K, v=V, o=O, lse=L, B=1, H=2, Nq=16, Nkv=16, d=64, scale=0.125,
                causal=0, stream=None, in_dtype=binding.FA_F16, o_dtype=binding.FA_F32)
    args.update(kw)
    return binding.fa_fwd(**args)


def test_library_builds_and_loads():
    assert fa_build.build().endswith("libfa_b200.so")
    lib = binding.library()
    assert lib.fa_version() == 100


def test_every_declared_symbol_is_exported():
    declared = binding.declared_functions()
    assert len(declared) >= 9
    nm = subprocess.run(["nm", "-D", "--defined-only", fa_build.LIB_PATH],
                        capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in nm.splitlines() if " T " in line}
    missing = [f for f in declared if f not in exported]
    assert not missing, f"declared but not exported: {missing}"
    lib = binding.library()
    for f in declared:
        assert hasattr(lib, f)


def test_status_strings():
    for code in range(7):
        assert binding.status_string(code) != "unknown status"
    assert binding.status_string(99) == "unknown status"


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), binding.FA_ERR_INVALID_ARG),
    (dict(k=None), binding.FA_ERR_INVALID_ARG),
    (dict(v=None), binding.FA_ERR_INVALID_ARG),
    (dict(o=None), binding.FA_ERR_INVALID_ARG),
    (dict(B=0), binding.FA_ERR_INVALID_ARG),
    (dict(H=-1), binding.FA_ERR_INVALID_ARG),
    (dict(Nq=0), binding.FA_ERR_INVALID_ARG),
    (dict(Nkv=0), binding.FA_ERR_INVALID_ARG),
    (dict(B=1 << 16, H=1 << 16), binding.FA_ERR_INVALID_ARG),
    (dict(causal=2), binding.FA_ERR_INVALID_ARG),
    (dict(scale=math.nan), binding.FA_ERR_INVALID_ARG),
    (dict(scale=math.inf), binding.FA_ERR_INVALID_ARG),
    (dict(in_dtype=binding.FA_F32), binding.FA_ERR_INVALID_ARG),
    (dict(o_dtype=7), binding.FA_ERR_INVALID_ARG),
    (dict(in_dtype=binding.FA_F16, o_dtype=binding.FA_BF16), binding.FA_ERR_UNSUPPORTED),
    (dict(d=96), binding.FA_ERR_UNSUPPORTED),
    (dict(d=256), binding.FA_ERR_UNSUPPORTED),
    (dict(q=Q + 8), binding.FA_ERR_INVALID_ARG),
    (dict(k=K + 2), binding.FA_ERR_INVALID_ARG),
    (dict(o=O + 4), binding.FA_ERR_INVALID_ARG),
    (dict(lse=L + 2), binding.FA_ERR_INVALID_ARG),
    (dict(o=Q), binding.FA_ERR_INVALID_ARG),                 # O overlaps Q
    (dict(o=K + 512), binding.FA_ERR_INVALID_ARG),           # O inside K
    (dict(lse=O + 64), binding.FA_ERR_INVALID_ARG),          # LSE inside O
    (dict(lse=V), binding.FA_ERR_INVALID_ARG),               # LSE on V
])
def test_argument_checks(kw, code):
    assert _fwd(**kw) == code


def test_prefill_and_decode_entry_checks():
    lib = binding
    assert lib.fa_fwd_prefill(Q, K, V, O, L, 1, 1, 4, 4, 64, 0.1, 0, None, 0, 2, -1) == \
        binding.FA_ERR_INVALID_ARG
    for ctas, splits in ((-1, 0), (0, -1), (0, 65)):
        assert lib.fa_fwd_prefill_split(Q, K, V, O, L, 1, 1, 4, 4, 64, 0.1, 0, None, 0, 2,
                                        ctas, splits) == binding.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_decode(Q, K, V, O, L, 1, 1, 4, 64, 0.1, None, 0, 2, -1) == \
        binding.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_decode(None, K, V, O, L, 1, 1, 4, 64, 0.1, None, 0, 2, 0) == \
        binding.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_decode(Q, K, V, O, L, 1, 1, 4, 80, 0.1, None, 0, 2, 0) == \
        binding.FA_ERR_UNSUPPORTED


def test_prefill_split_choice_is_host_arithmetic():
    ns = binding.prefill_num_splits
    # at least one unit (pair of 128-row Q tiles of one head) per SM: never split
    assert ns(1, 32, 8192, 8192, 128, True, 148) == 1
    assert ns(3, 1, 148 * 256, 148 * 256, 64, False, 148) == 1
    assert ns(1, 148, 256, 256, 128, False, 148) == 1
    # one head of 16k causal tokens on 148 SMs: 64 units, the longest 128 K/V tiles
    assert 2 <= ns(1, 1, 16384, 16384, 128, True, 148) <= 8
    # many short units: the split's fixed cost is not worth it
    assert ns(2, 8, 2048, 2048, 64, True, 148) == 1
    # where the split would take two parts, a causal launch runs unsplit as interleaved-K/V
    # units instead (no combine launch); from three parts on the split stays
    assert ns(1, 8, 4096, 4096, 128, True, 148) == 1
    assert ns(2, 4, 4096, 4096, 64, True, 148) == 1
    assert ns(1, 2, 8192, 8192, 128, True, 148) >= 3
    assert ns(1, 4, 4096, 4096, 128, True, 148) >= 3
    # never more parts than K/V tiles
    assert ns(1, 1, 300, 200, 128, False, 148) <= 2
    for args in ((0, 1, 4, 4, 64, 0, 148), (1, 1, 4, 4, 96, 0, 148), (1, 1, 4, 4, 64, 2, 148),
                 (1, 1, 4, 4, 64, 0, -1)):
        out = ctypes.c_int(0)
        assert binding.library().fa_prefill_num_splits(*args, ctypes.byref(out)) == \
            binding.FA_ERR_INVALID_ARG
    assert binding.library().fa_prefill_num_splits(1, 1, 4, 4, 64, 0, 148, None) == \
        binding.FA_ERR_INVALID_ARG


def test_decode_workspace_size_formula():
    # 16 partial records (one per consumer warp) per CTA per head segment, d+1 floats each.
    B, H, Nkv, d, G = 16, 32, 32768, 128, 148
    chunks = B * H * ((Nkv + 63) // 64)
    per_cta = -(-chunks // G)
    max_seg = -(-per_cta // ((Nkv + 63) // 64)) + 1
    assert binding.fa_decode_workspace_bytes(B, H, Nkv, d, G) == G * max_seg * 16 * (d + 1) * 4
    assert binding.fa_decode_workspace_bytes(1, 1, 10, 64, 5) == 1 * 2 * 16 * 65 * 4


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_valid_call_without_device_reports_cuda_error():
    assert _fwd() == binding.FA_ERR_CUDA
    assert binding.library().fa_last_cuda_error() != 0


# Every entry point that reaches the device, called with valid arguments in a process that
# sees no CUDA device: each must return FA_ERR_CUDA and leave the CUDA error code for
# fa_get_last_cuda_error, which clears it.  No device is visible, so nothing can launch.
_NO_DEVICE_SCRIPT = r"""
import ctypes, json, sys
sys.path.insert(0, sys.argv[1])
from exact_io_aware_59_b200 import binding as b
A = 1 << 20
Q, K, V, O, L = A, 2 * A, 3 * A, 4 * A, 5 * A
lib = b.library()
calls = {
    "fa_fwd": lambda: b.fa_fwd(Q, K, V, O, L, 1, 2, 16, 16, 64, 0.125, 0, None, 0, 2),
    "fa_fwd_prefill": lambda: b.fa_fwd_prefill(Q, K, V, O, L, 1, 2, 16, 16, 64, 0.125, 1, None,
                                               0, 2, 0),
    "fa_fwd_prefill_split": lambda: b.fa_fwd_prefill_split(Q, K, V, O, L, 1, 2, 600, 600, 64,
                                                           0.125, 1, None, 0, 2, 0, 3),
    "fa_prefill_num_splits": lambda: lib.fa_prefill_num_splits(1, 1, 9000, 9000, 128, 1, 0,
                                                               ctypes.byref(ctypes.c_int(0))),
    "fa_fwd_decode": lambda: b.fa_fwd_decode(Q, K, V, O, L, 1, 2, 16, 64, 0.125, None, 0, 2, 0),
    "fa_fwd_decode_noalloc": lambda: b.fa_fwd_decode_noalloc(Q, K, V, O, L, 1, 2, 16, 64, 0.125,
                                                             None, 0, 2, 0),
    "fa_fwd_fp8": lambda: b.fa_fwd_fp8(Q, K, V, O, L, 1, 1, 4, 4, 128, 0.1, 0, None, 1.0, 1.0, 1,
                                       2),
    "fa_fwd_varlen": lambda: b.fa_fwd_varlen(Q, K, V, O, L, L + 4096, L + 8192, 2, 2, 100, 100,
                                             60, 60, 64, 0.1, 1, None, 0, 2),
    "fa_fwd_decode_paged": lambda: b.fa_fwd_decode_paged(Q, K, V, L + 64, L + 128, O, L, 1, 1,
                                                         64, 16, 4, 8, 0.1, None, 0, 2, 0),
    "fa_bwd": lambda: b.fa_bwd(Q, K, V, O, L, Q + 4096, O + 4096, O + 8192, O + 12288,
                               O + 65536, 128 * 520, 1, 1, 4, 4, 128, 0.1, 0, None, 1),
    "fa_bwd_varlen": lambda: b.fa_bwd_varlen(Q, K, V, O, L, Q + 4096, O + 4096, O + 8192,
                                             O + 12288, 6 * A, A, 7 * A, 7 * A + 64, 1, 1, 4, 4,
                                             4, 4, 128, 0.1, 1, None, 1),
    "fa_quantize_e4m3": lambda: b.fa_quantize_e4m3(Q, 1, 2, 100, 128, O, L, None),
    "fa_fwd_fp8_quant": lambda: b.fa_fwd_fp8_quant(Q, K, V, O, L, 1, 2, 16, 16, 128, 0.1, 1,
                                                   None, 1, 2),
    "fa_device_status": lambda: lib.fa_device_status(ctypes.byref(ctypes.c_int(0)), 0),
    "fa_selftest_wait_timeout": lambda: lib.fa_selftest_wait_timeout(None),
    "fa_release_workspace": lambda: lib.fa_release_workspace(),
    "fa_decode_workspace_bytes": lambda: lib.fa_decode_workspace_bytes(
        1, 1, 64, 64, 0, ctypes.byref(ctypes.c_size_t(0))),
}
out = {}
for name, fn in calls.items():
    rc = int(fn())
    err = b.fa_get_last_cuda_error()
    out[name] = [rc, err, b.fa_get_last_cuda_error()]
print(json.dumps(out))
"""


def test_every_entry_point_reports_its_cuda_error():
    import json
    import os
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-c", _NO_DEVICE_SCRIPT, root], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    out = json.loads(r.stdout.strip().splitlines()[-1])
    codes = set()
    for name, (rc, err, err_after) in out.items():
        assert rc == binding.FA_ERR_CUDA, (name, rc)
        assert err != 0, name                # the cudaError_t behind FA_ERR_CUDA
        assert err_after == 0, name          # reading it cleared it
        codes.add(err)
    assert len(codes) == 1                   # the same "no device" error everywhere


def test_get_last_cuda_error_checks_its_pointer():
    assert binding.library().fa_get_last_cuda_error(None) == binding.FA_ERR_INVALID_ARG


def test_binding_rejects_host_tensors():
    q = torch.zeros(1, 1, 4, 64, dtype=torch.float16)
    with pytest.raises(ValueError):
        binding.attention(q, q, q)


def _paged(**kw):
    a = dict(q=Q, kc=K, vc=V, table=L + 64, lens=L + 128, o=O, lse=L, B=1, H=1, d=64,
             page_size=16, max_pages=4, num_pages=8, scale=0.1, stream=None, in_dtype=0,
             o_dtype=2, num_splits=0)
    a.update(kw)
    return binding.fa_fwd_decode_paged(a["q"], a["kc"], a["vc"], a["table"], a["lens"], a["o"],
                                       a["lse"], a["B"], a["H"], a["d"], a["page_size"],
                                       a["max_pages"], a["num_pages"], a["scale"], a["stream"],
                                       a["in_dtype"], a["o_dtype"], a["num_splits"])


@pytest.mark.parametrize("kw,code", [
    (dict(table=None), binding.FA_ERR_INVALID_ARG),
    (dict(lens=None), binding.FA_ERR_INVALID_ARG),
    (dict(kc=None), binding.FA_ERR_INVALID_ARG),
    (dict(page_size=8), binding.FA_ERR_INVALID_ARG),      # below 16
    (dict(page_size=48), binding.FA_ERR_INVALID_ARG),     # not a power of two
    (dict(page_size=2048), binding.FA_ERR_INVALID_ARG),
    (dict(max_pages=0), binding.FA_ERR_INVALID_ARG),
    (dict(num_pages=0), binding.FA_ERR_INVALID_ARG),
    (dict(max_pages=1 << 22, page_size=1024), binding.FA_ERR_INVALID_ARG),  # > 2^31 keys
    (dict(num_splits=-1), binding.FA_ERR_INVALID_ARG),
    (dict(table=L + 66), binding.FA_ERR_INVALID_ARG),     # misaligned int32 table
    (dict(d=96), binding.FA_ERR_UNSUPPORTED),
    (dict(in_dtype=0, o_dtype=1), binding.FA_ERR_UNSUPPORTED),
    (dict(o=K), binding.FA_ERR_INVALID_ARG),              # O on the key cache
])
def test_paged_decode_argument_checks(kw, code):
    assert _paged(**kw) == code


def _varlen(**kw):
    a = dict(q=Q, k=K, v=V, o=O, lse=L, cq=L + 4096, ck=L + 8192, B=2, H=2, tq=100, tk=100,
             mq=60, mk=60, d=64, scale=0.1, causal=1, stream=None, in_dtype=0, o_dtype=2)
    a.update(kw)
    return binding.fa_fwd_varlen(a["q"], a["k"], a["v"], a["o"], a["lse"], a["cq"], a["ck"],
                                 a["B"], a["H"], a["tq"], a["tk"], a["mq"], a["mk"], a["d"],
                                 a["scale"], a["causal"], a["stream"], a["in_dtype"],
                                 a["o_dtype"])


@pytest.mark.parametrize("kw,code", [
    (dict(cq=None), binding.FA_ERR_INVALID_ARG),
    (dict(ck=None), binding.FA_ERR_INVALID_ARG),
    (dict(B=0), binding.FA_ERR_INVALID_ARG),
    (dict(tq=0), binding.FA_ERR_INVALID_ARG),
    (dict(mk=0), binding.FA_ERR_INVALID_ARG),
    (dict(mq=101), binding.FA_ERR_INVALID_ARG),        # longer than the whole batch
    (dict(causal=3), binding.FA_ERR_INVALID_ARG),
    (dict(cq=L + 4098), binding.FA_ERR_INVALID_ARG),   # misaligned int32 offsets
    (dict(d=32), binding.FA_ERR_UNSUPPORTED),
    (dict(o=Q), binding.FA_ERR_INVALID_ARG),           # O on Q
])
def test_varlen_argument_checks(kw, code):
    assert _varlen(**kw) == code


def test_fp8_entry_checks():
    f = binding.fa_fwd_fp8
    args = dict(q8=Q, k8=K, v=V, o=O, lse=L, B=1, H=1, Nq=4, Nkv=4, d=128, scale=0.1, causal=0,
                stream=None, qs=1.0, ks=1.0, vd=1, od=2)

    def call(**kw):
        a = dict(args)
        a.update(kw)
        return f(a["q8"], a["k8"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["Nq"], a["Nkv"],
                 a["d"], a["scale"], a["causal"], a["stream"], a["qs"], a["ks"], a["vd"], a["od"])

    assert call(d=64) == binding.FA_ERR_UNSUPPORTED
    assert call(q8=None) == binding.FA_ERR_INVALID_ARG
    assert call(qs=math.inf) == binding.FA_ERR_INVALID_ARG
    assert call(vd=2) == binding.FA_ERR_INVALID_ARG          # V must be 16-bit
    assert call(vd=0, od=1) == binding.FA_ERR_UNSUPPORTED     # 16-bit O must be V's type
    assert call(k8=K + 8) == binding.FA_ERR_INVALID_ARG       # misaligned


def test_backward_entry_checks():
    """fa_bwd refuses bad arguments on the host, before touching any device."""
    ws_ok = 1 * 1 * 128 * 520
    args = dict(q=Q, k=K, v=V, o=O, lse=L, do=Q + 4096, dq=O + 4096, dk=O + 8192, dv=O + 12288,
                ws=O + 65536, wsb=ws_ok, B=1, H=1, Nq=4, Nkv=4, d=128, scale=0.1, causal=0,
                stream=None, dt=1)

    def call(**kw):
        a = dict(args)
        a.update(kw)
        return binding.fa_bwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["do"], a["dq"], a["dk"],
                              a["dv"], a["ws"], a["wsb"], a["B"], a["H"], a["Nq"], a["Nkv"],
                              a["d"], a["scale"], a["causal"], a["stream"], a["dt"])

    assert call(d=96) == binding.FA_ERR_UNSUPPORTED
    assert call(lse=None) == binding.FA_ERR_INVALID_ARG
    assert call(ws=None) == binding.FA_ERR_INVALID_ARG
    assert call(wsb=ws_ok - 16) == binding.FA_ERR_INVALID_ARG   # workspace too small
    assert call(Nq=0) == binding.FA_ERR_INVALID_ARG
    assert call(causal=2) == binding.FA_ERR_INVALID_ARG
    assert call(dt=2) == binding.FA_ERR_INVALID_ARG             # fp32 inputs
    assert call(scale=math.nan) == binding.FA_ERR_INVALID_ARG
    assert call(dk=O + 8200) == binding.FA_ERR_INVALID_ARG      # misaligned
    assert call(dq=Q) == binding.FA_ERR_INVALID_ARG             # output overlaps an input
    assert call(dv=O + 8192) == binding.FA_ERR_INVALID_ARG      # two outputs overlap
    assert binding.fa_bwd_workspace_bytes(2, 3, 65, 128) == 2 * 3 * 128 * 520
    assert binding.fa_bwd_workspace_bytes(1, 1, 129, 128) == 256 * 520
    assert binding.fa_bwd_workspace_bytes(1, 1, 64, 64) == 128 * (8 + 4 * 64)
    with pytest.raises(binding.FaError):
        binding.fa_bwd_workspace_bytes(1, 1, 64, 96)


def test_backward_varlen_entry_checks():
    """fa_bwd_varlen refuses bad arguments on the host, before touching any device."""
    B, H, tq, tk, d = 2, 3, 300, 400, 128
    rows_max = (tq + 128 * B + 127) // 128 * 128
    need = H * rows_max * (8 + 4 * d) + 16 + 16 * B + ((4 * (B + 1) + 15) // 16) * 16 + 4 * B * 2
    assert binding.fa_bwd_varlen_workspace_bytes(B, H, tq, 200, d) == need   # 2 key tiles
    with pytest.raises(binding.FaError):
        binding.fa_bwd_varlen_workspace_bytes(B, H, tq, 200, 96)
    A_ = 1 << 24
    args = dict(q=A_, k=2 * A_, v=3 * A_, o=4 * A_, lse=5 * A_, do=6 * A_, dq=7 * A_, dk=8 * A_,
                dv=9 * A_, ws=10 * A_, wsb=need, cq=11 * A_, ck=11 * A_ + 64, B=B, H=H, tq=tq,
                tk=tk, mq=200, mk=200, d=d, scale=0.1, causal=1, stream=None, dt=1)

    def call(**kw):
        a = dict(args)
        a.update(kw)
        return binding.fa_bwd_varlen(a["q"], a["k"], a["v"], a["o"], a["lse"], a["do"], a["dq"],
                                     a["dk"], a["dv"], a["ws"], a["wsb"], a["cq"], a["ck"], a["B"],
                                     a["H"], a["tq"], a["tk"], a["mq"], a["mk"], a["d"],
                                     a["scale"], a["causal"], a["stream"], a["dt"])

    assert call(d=96) == binding.FA_ERR_UNSUPPORTED
    assert call(cq=None) == binding.FA_ERR_INVALID_ARG
    assert call(wsb=need - 4) == binding.FA_ERR_INVALID_ARG      # workspace too small
    assert call(mq=tq + 1) == binding.FA_ERR_INVALID_ARG         # longer than the batch
    assert call(B=0) == binding.FA_ERR_INVALID_ARG
    assert call(causal=2) == binding.FA_ERR_INVALID_ARG
    assert call(dt=2) == binding.FA_ERR_INVALID_ARG
    assert call(scale=math.inf) == binding.FA_ERR_INVALID_ARG
    assert call(dk=8 * A_ + 8) == binding.FA_ERR_INVALID_ARG      # misaligned
    assert call(ck=11 * A_ + 2) == binding.FA_ERR_INVALID_ARG     # misaligned offsets
    assert call(dq=A_) == binding.FA_ERR_INVALID_ARG              # output overlaps an input
    assert call(ws=11 * A_ - 64) == binding.FA_ERR_INVALID_ARG    # workspace overlaps cu_seqlens


def _declared_param_counts():
    """Parameter count of every function include/fa.h declares."""
    import re
    text = open(binding.HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = {}
    for m in re.finditer(r"^\s*(?:const\s+)?\w+\s*\*?\s*(fa_\w+)\s*\(([^)]*)\)\s*;", text, flags=re.M | re.S):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else len(params.split(","))
    return out


def test_binding_signatures_match_the_header():
    """Every ctypes signature has as many arguments as the C declaration (a binding that
    drifted from the header would pass garbage silently)."""
    counts = _declared_param_counts()
    assert set(counts) == set(binding.declared_functions())
    for name, argtypes in binding._SIGNATURES.items():
        assert name in counts, name
        assert len(argtypes) == counts[name], (name, len(argtypes), counts[name])


def test_quantize_entry_checks():
    q = binding.fa_quantize_e4m3
    assert q(Q, 1, 2, 100, 64, O, L, None) == binding.FA_ERR_UNSUPPORTED      # d must be 128
    assert q(None, 1, 2, 100, 128, O, L, None) == binding.FA_ERR_INVALID_ARG
    assert q(Q, 2, 2, 100, 128, O, L, None) == binding.FA_ERR_INVALID_ARG     # fp32 input
    assert q(Q, 1, 0, 100, 128, O, L, None) == binding.FA_ERR_INVALID_ARG
    assert q(Q + 8, 1, 2, 100, 128, O, L, None) == binding.FA_ERR_INVALID_ARG  # misaligned
    assert q(Q, 1, 2, 100, 128, Q + 1024, L, None) == binding.FA_ERR_INVALID_ARG  # codes on x
