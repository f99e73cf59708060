"""CPU checks of the C-ABI boundary: the library loads, exports every symbol the
header declares, and rejects bad arguments before enqueuing anything (these
calls return from validation, so no GPU is touched)."""
import ctypes
import os
import re

import pytest

from exact_attention_108_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fattn.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fattn_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(binding.LIB_PATH):
        from exact_attention_108_b200 import build
        build.build()
    return binding.load()


def test_header_declares_the_expected_entry_points():
    assert set(_declared_functions()) == set(binding.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for s in range(6):
        assert binding.status_string(s)
    assert binding.status_string(0) == "ok"
    assert lib.fattn_version() == 0x000200


P = 1 << 20  # a fake, 16-byte aligned "device" address; never dereferenced


def _fwd(lib, q=P, k=P, v=P, o=P, lse=P, B=1, H=1, N=128, d=64, causal=0, scale=0.125):
    return lib.fattn_fwd(q, k, v, o, lse, B, H, N, d, causal, scale, None)


def test_fwd_validation(lib):
    assert _fwd(lib, q=None) == binding.FATTN_ERR_INVALID_ARG
    assert _fwd(lib, lse=None) == binding.FATTN_ERR_INVALID_ARG
    assert _fwd(lib, B=0) == binding.FATTN_ERR_INVALID_ARG
    assert _fwd(lib, H=-1) == binding.FATTN_ERR_INVALID_ARG
    assert _fwd(lib, N=0) == binding.FATTN_ERR_INVALID_ARG
    assert _fwd(lib, d=80) == binding.FATTN_ERR_UNSUPPORTED
    assert _fwd(lib, d=512) == binding.FATTN_ERR_UNSUPPORTED
    assert _fwd(lib, d=16) == binding.FATTN_ERR_UNSUPPORTED
    assert _fwd(lib, B=1 << 14, H=1 << 10, N=1 << 8) == binding.FATTN_ERR_UNSUPPORTED  # 2^32 rows
    # 2^23 heads of 129 rows: under 2^31 rows, but 2^31 once each head is padded to whole tiles
    assert _fwd(lib, B=1 << 13, H=1 << 10, N=129) == binding.FATTN_ERR_UNSUPPORTED
    assert _fwd(lib, scale=float("inf")) == binding.FATTN_ERR_INVALID_ARG
    assert _fwd(lib, scale=float("nan")) == binding.FATTN_ERR_INVALID_ARG
    assert _fwd(lib, causal=2) == binding.FATTN_ERR_INVALID_ARG
    assert _fwd(lib, k=P + 8) == binding.FATTN_ERR_ALIGNMENT
    assert _fwd(lib, lse=P + 4) == binding.FATTN_ERR_ALIGNMENT


def test_workspace_size(lib):
    def a256(x):
        return (x + 255) // 256 * 256
    # D and LSE*log2(e) per head padded to whole 128-row tiles, then the fp32 dQ accumulator
    for (B, H, N, d) in [(1, 1, 128, 64), (4, 32, 4096, 128), (3, 5, 384, 128), (1, 1, 100, 64), (2, 3, 200, 128),
                         (1, 2, 300, 32), (2, 1, 129, 96)]:
        padded = B * H * ((N + 127) // 128 * 128)
        assert lib.fattn_bwd_workspace_size(B, H, N, d) == 2 * a256(padded * 4) + a256(B * H * N * d * 4)
    assert lib.fattn_bwd_workspace_size(1, 1, 128, 80) == 0
    assert lib.fattn_bwd_workspace_size(1, 1, 0, 64) == 0


def _bwd(lib, ws=P, ws_bytes=None, d=64, N=128, **kw):
    if ws_bytes is None:
        ws_bytes = lib.fattn_bwd_workspace_size(1, 1, N, d) if d in (32, 64, 96, 128) else 1 << 30
    args = dict(q=P, k=P, v=P, o=P, do=P, lse=P, dq=P, dk=P, dv=P)
    args.update(kw)
    return lib.fattn_bwd(args["q"], args["k"], args["v"], args["o"], args["do"], args["lse"], args["dq"],
                         args["dk"], args["dv"], 1, 1, N, d, 0, 0.125, ws, ws_bytes, None)


def test_bwd_validation(lib):
    assert _bwd(lib, do=None) == binding.FATTN_ERR_INVALID_ARG
    assert _bwd(lib, ws=None) == binding.FATTN_ERR_INVALID_ARG
    assert _bwd(lib, ws_bytes=16) == binding.FATTN_ERR_INVALID_ARG
    assert _bwd(lib, d=48) == binding.FATTN_ERR_UNSUPPORTED
    assert _bwd(lib, d=256) == binding.FATTN_ERR_UNSUPPORTED  # d = 256: forward only
    assert lib.fattn_bwd_workspace_size(1, 1, 128, 256) == 0
    assert _bwd(lib, N=200, ws_bytes=lib.fattn_bwd_workspace_size(1, 1, 200, 64) - 16) == binding.FATTN_ERR_INVALID_ARG
    assert _bwd(lib, dq=P + 2) == binding.FATTN_ERR_ALIGNMENT
    assert _bwd(lib, ws=P + 16) == binding.FATTN_ERR_ALIGNMENT  # workspace wants 256 bytes


def test_python_binding_rejects_host_tensors():
    import torch
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        binding.fwd(q, q, q)


# ------------------------------------------------------------- general forms
def test_param_structs_match_the_c_layout(tmp_path):
    """The ctypes mirrors of fattn_fwd_params / fattn_bwd_params have the C layout
    (offsets printed by a C program compiled against include/fattn.h)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    fields = {"fattn_fwd_params": binding.FwdParams, "fattn_bwd_params": binding.BwdParams,
              "fattn_decode_params": binding.DecodeParams}
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "fattn.h"', "int main(void) {"]
    for cname, py in fields.items():
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for f, _ in py._fields_:
            lines.append(f'  printf("{cname} {f} %zu\\n", offsetof({cname}, {f}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run([cc, "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    got = {tuple(x.split()[:2]): int(x.split()[2]) for x in out if x}
    for cname, py in fields.items():
        assert got[(cname, "size")] == ctypes.sizeof(py)
        for f, _ in py._fields_:
            assert got[(cname, f)] == getattr(py, f).offset, (cname, f)


def _fwd_ex(lib, **kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, B=1, H=4, H_kv=2, N_q=100, N_k=300, d=128, causal=1, scale=0.1,
             dropout_p=0.0, seed=0, offset=0)
    a.update(kw)
    p = binding.FwdParams(*[a[f] for f, _ in binding.FwdParams._fields_])
    return lib.fattn_fwd_ex(ctypes.byref(p), None)


def test_fwd_ex_validation(lib):
    assert lib.fattn_fwd_ex(None, None) == binding.FATTN_ERR_INVALID_ARG
    assert _fwd_ex(lib, H_kv=3) == binding.FATTN_ERR_INVALID_ARG      # H not a multiple of H_kv
    assert _fwd_ex(lib, H_kv=0) == binding.FATTN_ERR_INVALID_ARG
    assert _fwd_ex(lib, N_q=0) == binding.FATTN_ERR_INVALID_ARG
    assert _fwd_ex(lib, N_k=-1) == binding.FATTN_ERR_INVALID_ARG
    assert _fwd_ex(lib, dropout_p=1.0) == binding.FATTN_ERR_INVALID_ARG
    assert _fwd_ex(lib, dropout_p=-0.1) == binding.FATTN_ERR_INVALID_ARG
    assert _fwd_ex(lib, dropout_p=float("nan")) == binding.FATTN_ERR_INVALID_ARG
    assert _fwd_ex(lib, d=512) == binding.FATTN_ERR_UNSUPPORTED
    assert _fwd_ex(lib, d=256, dropout_p=0.1) == binding.FATTN_ERR_UNSUPPORTED  # d = 256: no dropout
    assert _fwd_ex(lib, B=1 << 14, H=1 << 10, H_kv=1, N_q=128, N_k=128) == binding.FATTN_ERR_UNSUPPORTED
    assert _fwd_ex(lib, B=1 << 14, H=1 << 10, H_kv=1 << 10, N_q=1, N_k=128) == binding.FATTN_ERR_UNSUPPORTED
    assert _fwd_ex(lib, v=P + 8) == binding.FATTN_ERR_ALIGNMENT
    assert _fwd_ex(lib, o=None) == binding.FATTN_ERR_INVALID_ARG


def _bwd_params(**kw):
    a = dict(q=P, k=P, v=P, o=P, dout=P, lse=P, dq=P, dk=P, dv=P, B=2, H=4, H_kv=1, N_q=200, N_k=333, d=64,
             causal=1, scale=0.1, dropout_p=0.2, seed=7, offset=3, deterministic=0, workspace=P,
             workspace_bytes=0)
    a.update(kw)
    return binding.BwdParams(*[a[f] for f, _ in binding.BwdParams._fields_])


def test_bwd_ex_workspace_size_and_validation(lib):
    def a256(x):
        return (x + 255) // 256 * 256
    for det in (0, 1):
        p = _bwd_params(deterministic=det)
        stat = a256(2 * 4 * 256 * 4)  # B*H heads, N_q padded to 256 rows
        acc = 0 if det else a256(2 * 4 * 200 * 64 * 4)
        assert lib.fattn_bwd_ex_workspace_size(ctypes.byref(p)) == 2 * stat + acc
    assert lib.fattn_bwd_ex_workspace_size(ctypes.byref(_bwd_params(H_kv=3))) == 0
    need = lib.fattn_bwd_ex_workspace_size(ctypes.byref(_bwd_params()))
    assert lib.fattn_bwd_ex(ctypes.byref(_bwd_params(workspace_bytes=need - 1)), None) == binding.FATTN_ERR_INVALID_ARG
    assert lib.fattn_bwd_ex(ctypes.byref(_bwd_params(workspace_bytes=need, workspace=P + 16)), None) == \
        binding.FATTN_ERR_ALIGNMENT
    assert lib.fattn_bwd_ex(ctypes.byref(_bwd_params(workspace_bytes=need, deterministic=2)), None) == \
        binding.FATTN_ERR_INVALID_ARG
    assert lib.fattn_bwd_ex(ctypes.byref(_bwd_params(workspace_bytes=need, dq=None)), None) == \
        binding.FATTN_ERR_INVALID_ARG
    assert lib.fattn_bwd_ex(None, None) == binding.FATTN_ERR_INVALID_ARG


def _dec(lib, **kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, B=2, H=8, H_kv=2, N_q=1, N_k=1000, N_k_cap=1024, d=128, causal=1,
             scale=0.1, num_splits=0, workspace=None, workspace_bytes=0)
    a.update(kw)
    p = binding.DecodeParams(*[a[f] for f, _ in binding.DecodeParams._fields_])
    return lib.fattn_decode(ctypes.byref(p), None)


def test_decode_validation(lib):
    assert lib.fattn_decode(None, None) == binding.FATTN_ERR_INVALID_ARG
    assert _dec(lib, N_k_cap=999) == binding.FATTN_ERR_INVALID_ARG    # cache smaller than N_k
    assert _dec(lib, H_kv=3) == binding.FATTN_ERR_INVALID_ARG
    assert _dec(lib, num_splits=-1) == binding.FATTN_ERR_INVALID_ARG
    assert _dec(lib, causal=3) == binding.FATTN_ERR_INVALID_ARG
    assert _dec(lib, scale=float("inf")) == binding.FATTN_ERR_INVALID_ARG
    assert _dec(lib, d=48) == binding.FATTN_ERR_UNSUPPORTED
    assert _dec(lib, q=P + 4) == binding.FATTN_ERR_ALIGNMENT
