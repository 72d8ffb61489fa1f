"""CPU checks of the C ABI: the library loads, exports every declared symbol,
its argument structs match the header's layout, and host-side validation
rejects bad arguments before anything is launched (no GPU needed: every call
here fails validation, which happens before the first CUDA runtime call)."""
import ctypes
import os
import re
import subprocess

import pytest

from gated_delta_rule_148_b200 import kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(kda_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    lib = kda.load()
    declared = _declared_functions()
    assert set(kda.EXPORTED) <= set(declared)
    out = subprocess.run(["nm", "-D", "--defined-only", kda.library_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\b(kda_\w+)$", out, flags=re.M))
    missing = [n for n in declared if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    for name in declared:
        assert hasattr(lib, name)
    assert lib.kda_version() >> 16 == 1


def test_struct_layout_matches_header(tmp_path):
    prog = tmp_path / "layout.c"
    fields_p = [f[0] for f in kda.PrefillArgs._fields_]
    fields_d = [f[0] for f in kda.DecodeArgs._fields_]
    fields_c = [f[0] for f in kda.ConvArgs._fields_]
    fields_b = [f[0] for f in kda.BackwardArgs._fields_]
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "kda.h"', 'int main(void){']
    lines.append('printf("P %zu\\n", sizeof(kda_prefill_args));')
    for f in fields_p:
        lines.append(f'printf("P.{f} %zu\\n", offsetof(kda_prefill_args, {f}));')
    lines.append('printf("D %zu\\n", sizeof(kda_decode_args));')
    for f in fields_d:
        lines.append(f'printf("D.{f} %zu\\n", offsetof(kda_decode_args, {f}));')
    lines.append('printf("C %zu\\n", sizeof(kda_conv_args));')
    for f in fields_c:
        lines.append(f'printf("C.{f} %zu\\n", offsetof(kda_conv_args, {f}));')
    lines.append('printf("B %zu\\n", sizeof(kda_backward_args));')
    for f in fields_b:
        lines.append(f'printf("B.{f} %zu\\n", offsetof(kda_backward_args, {f}));')
    lines.append("return 0;}")
    prog.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(prog),
                           "-o", str(exe)])
    got = dict(line.split() for line in subprocess.check_output([str(exe)], text=True).splitlines())
    assert int(got["P"]) == ctypes.sizeof(kda.PrefillArgs)
    assert int(got["D"]) == ctypes.sizeof(kda.DecodeArgs)
    for f in fields_p:
        assert int(got[f"P.{f}"]) == getattr(kda.PrefillArgs, f).offset, f
    for f in fields_d:
        assert int(got[f"D.{f}"]) == getattr(kda.DecodeArgs, f).offset, f
    assert int(got["C"]) == ctypes.sizeof(kda.ConvArgs)
    for f in fields_c:
        assert int(got[f"C.{f}"]) == getattr(kda.ConvArgs, f).offset, f
    assert int(got["B"]) == ctypes.sizeof(kda.BackwardArgs)
    for f in fields_b:
        assert int(got[f"B.{f}"]) == getattr(kda.BackwardArgs, f).offset, f


def test_status_strings():
    for code in range(6):
        assert kda.status_string(code).startswith("KDA_")


# Fake device addresses: validation rejects these calls before any CUDA call,
# so nothing is ever dereferenced.
BASE = 0x7F0000000000
N, H, D, B = 256, 2, 64, 2


def _good_prefill():
    a = kda.PrefillArgs()
    a.dtype, a.num_seqs, a.total_tokens, a.H, a.dk, a.dv = kda.KDA_BF16, B, N, H, D, D
    sz = N * H * D * 2
    a.q, a.k, a.v = BASE, BASE + sz, BASE + 2 * sz
    a.log_alpha = BASE + 3 * sz
    a.beta = BASE + 3 * sz + N * H * D * 4
    a.cu_seqlens = a.beta + N * H * 4
    a.o = BASE + 0x100000000
    a.chunk = 64
    return a


def _call(a):
    return kda.load().kda_prefill(ctypes.byref(a), None)


@pytest.mark.parametrize("mutate,expect", [
    (lambda a: setattr(a, "dtype", 7), kda.KDA_ERR_INVALID_ARG),
    (lambda a: setattr(a, "H", 0), kda.KDA_ERR_INVALID_ARG),
    (lambda a: setattr(a, "num_seqs", -1), kda.KDA_ERR_INVALID_ARG),
    (lambda a: setattr(a, "dk", 96), kda.KDA_ERR_UNSUPPORTED),
    (lambda a: setattr(a, "dv", 256), kda.KDA_ERR_UNSUPPORTED),
    (lambda a: setattr(a, "chunk", 48), kda.KDA_ERR_UNSUPPORTED),
    (lambda a: setattr(a, "chunk", 128), kda.KDA_ERR_UNSUPPORTED),            # d = 64
    (lambda a: (setattr(a, "chunk", 256), setattr(a, "dtype", kda.KDA_F32)), kda.KDA_ERR_UNSUPPORTED),
    (lambda a: setattr(a, "chunk", 512), kda.KDA_ERR_UNSUPPORTED),
    (lambda a: setattr(a, "q", None), kda.KDA_ERR_INVALID_ARG),
    (lambda a: setattr(a, "o", None), kda.KDA_ERR_INVALID_ARG),
    (lambda a: setattr(a, "cu_seqlens", None), kda.KDA_ERR_INVALID_ARG),
    (lambda a: setattr(a, "q", BASE + 8), kda.KDA_ERR_INVALID_ARG),          # misaligned
    (lambda a: setattr(a, "log_alpha", a.log_alpha + 4), kda.KDA_ERR_INVALID_ARG),
    (lambda a: setattr(a, "o", a.k + 1024), kda.KDA_ERR_INVALID_ARG),          # o overlaps k
    (lambda a: setattr(a, "pad_mask", BASE + 0x200000000), kda.KDA_ERR_INVALID_ARG),  # no ws
    (lambda a: (setattr(a, "final_state", a.q)), kda.KDA_ERR_INVALID_ARG),     # aliases q
    (lambda a: (setattr(a, "num_seqs", 0)), kda.KDA_ERR_INVALID_ARG),          # N>0, no seqs
    (lambda a: setattr(a, "gate", 2), kda.KDA_ERR_INVALID_ARG),               # unknown layout
    (lambda a: (setattr(a, "gate", kda.KDA_GATE_HEAD),                        # head gate: 4-B
                setattr(a, "log_alpha", a.log_alpha + 2)), kda.KDA_ERR_INVALID_ARG),
    (lambda a: (setattr(a, "gate", kda.KDA_GATE_HEAD),                        # [N, H] gate
                setattr(a, "o", a.log_alpha + N * H * 4 - 64)), kda.KDA_ERR_INVALID_ARG),
], ids=["dtype", "H", "num_seqs", "dk", "dv", "chunk", "chunk128_d64", "chunk256_f32",
        "chunk512", "null_q", "null_o", "null_cu",
        "misaligned_q", "misaligned_la", "o_overlaps_k", "mask_without_ws", "state_aliases_q",
        "tokens_without_seqs", "gate_value", "head_gate_misaligned", "o_overlaps_head_gate"])
def test_prefill_rejects_bad_arguments(mutate, expect):
    a = _good_prefill()
    mutate(a)
    assert _call(a) == expect


def test_prefill_null_args_and_empty_batch():
    assert kda.load().kda_prefill(None, None) == kda.KDA_ERR_INVALID_ARG
    a = kda.PrefillArgs()
    a.dtype, a.num_seqs, a.total_tokens, a.H, a.dk, a.dv = kda.KDA_F32, 0, 0, 1, 64, 64
    assert _call(a) == kda.KDA_OK          # nothing to do, nothing launched


def test_workspace_size():
    a = kda.PrefillArgs()
    a.num_seqs = 8
    n = kda.load().kda_prefill_workspace_size(ctypes.byref(a))
    assert n >= 8 * 16 and n % 256 == 0
    assert kda.load().kda_prefill_workspace_size(None) == 0


def test_workspace_size_by_chunk():
    """bf16, d = 128: chunk 64 needs the 64-row items (74 752 bytes per chunk and head);
    chunks of 128 / 256 also need the merged items (164 352 and 360 960 bytes)."""
    a = kda.PrefillArgs()
    a.dtype, a.num_seqs, a.total_tokens, a.H, a.dk, a.dv = kda.KDA_BF16, 1, 131072, 32, 128, 128
    size = {}
    for c in (64, 128, 256):
        a.chunk = c
        size[c] = kda.load().kda_prefill_workspace_size(ctypes.byref(a))
    items64 = (131072 // 64 + 1) * 32 * 74752
    items128 = (131072 // 128 + 1) * 32 * 164352
    items256 = (131072 // 256 + 1) * 32 * 360960
    assert items64 < size[64] < items64 + 4096
    assert items64 + items128 < size[128] < items64 + items128 + 8192
    assert max(items64, items256) + items128 < size[256] < max(items64, items256) + items128 + 8192
    a.dtype = kda.KDA_F32
    assert kda.load().kda_prefill_workspace_size(ctypes.byref(a)) < 4096   # no tensor-core path


def _good_decode():
    a = kda.DecodeArgs()
    a.dtype, a.B, a.H, a.dk, a.dv = kda.KDA_BF16, 4, 2, 128, 128
    a.q, a.k, a.v = BASE, BASE + 0x10000, BASE + 0x20000
    a.log_alpha, a.beta = BASE + 0x30000, BASE + 0x40000
    a.state, a.o = BASE + 0x100000, BASE + 0x50000
    return a


@pytest.mark.parametrize("mutate,expect", [
    (lambda a: setattr(a, "dtype", 3), kda.KDA_ERR_INVALID_ARG),
    (lambda a: setattr(a, "dk", 32), kda.KDA_ERR_UNSUPPORTED),
    (lambda a: setattr(a, "state", None), kda.KDA_ERR_INVALID_ARG),
    (lambda a: setattr(a, "state", a.state + 4), kda.KDA_ERR_INVALID_ARG),
    (lambda a: setattr(a, "o", a.state + 64), kda.KDA_ERR_INVALID_ARG),
    (lambda a: setattr(a, "o", a.q + 2), kda.KDA_ERR_INVALID_ARG),
    (lambda a: setattr(a, "gate", -1), kda.KDA_ERR_INVALID_ARG),
], ids=["dtype", "dk", "null_state", "misaligned_state", "o_in_state", "o_overlaps_q",
        "gate_value"])
def test_decode_rejects_bad_arguments(mutate, expect):
    a = _good_decode()
    mutate(a)
    assert kda.load().kda_decode(ctypes.byref(a), None) == expect


def test_binding_refuses_host_tensors():
    import torch
    x = torch.zeros(4, 1, 64)
    with pytest.raises(TypeError):
        kda.decode(x, x, x, x, torch.zeros(4, 1), torch.zeros(4, 1, 64, 64))


def _good_conv():
    a = kda.ConvArgs()
    a.dtype, a.num_seqs, a.total_tokens, a.D, a.width = kda.KDA_BF16, 2, 256, 64, 4
    a.x, a.y = BASE, BASE + 0x100000
    a.weight, a.bias, a.cu_seqlens = BASE + 0x200000, BASE + 0x210000, BASE + 0x220000
    a.state_in, a.state_out = BASE + 0x230000, BASE + 0x240000
    return a


@pytest.mark.parametrize("mutate,expect", [
    (lambda a: setattr(a, "dtype", 5), kda.KDA_ERR_INVALID_ARG),
    (lambda a: setattr(a, "D", 60), kda.KDA_ERR_INVALID_ARG),           # not a multiple of 8
    (lambda a: setattr(a, "width", 5), kda.KDA_ERR_UNSUPPORTED),
    (lambda a: setattr(a, "width", 0), kda.KDA_ERR_UNSUPPORTED),
    (lambda a: setattr(a, "weight", None), kda.KDA_ERR_INVALID_ARG),
    (lambda a: setattr(a, "x", BASE + 4), kda.KDA_ERR_INVALID_ARG),      # misaligned
    (lambda a: setattr(a, "y", a.x + 64), kda.KDA_ERR_INVALID_ARG),      # y overlaps x
    (lambda a: setattr(a, "state_out", a.x), kda.KDA_ERR_INVALID_ARG),   # state over x
    (lambda a: setattr(a, "num_seqs", 0), kda.KDA_ERR_INVALID_ARG),      # tokens, no seqs
], ids=["dtype", "D", "width5", "width0", "null_weight", "misaligned_x", "y_overlaps_x",
        "state_over_x", "tokens_without_seqs"])
def test_conv_rejects_bad_arguments(mutate, expect):
    a = _good_conv()
    mutate(a)
    assert kda.load().kda_short_conv(ctypes.byref(a), None) == expect


def test_debug_fault_hook_rejects_unknown_bits_and_resets():
    lib = kda.load()
    assert lib.kda_debug_set_fault(1 << 7, 0) == kda.KDA_ERR_INVALID_ARG
    assert lib.kda_debug_set_fault(0, 0) == kda.KDA_OK
