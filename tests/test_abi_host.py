"""The C ABI without a GPU: the library loads, exports what include/bsfa.h
declares, and rejects bad arguments before making any CUDA call."""
import os
import re
import subprocess

import pytest

from threshold_gated_block_b200 import bsfa
from threshold_gated_block_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return bsfa.load()


def _declared():
    text = open(os.path.join(ROOT, "include", "bsfa.h")).read()
    return sorted(set(re.findall(r"^(?:bsfa_status|const char\*)\s+(bsfa_\w+)\(", text, flags=re.M)))


def test_header_declares_the_binding_names():
    assert _declared() == sorted(bsfa.EXPORTED)


def test_binding_signatures_match_the_header(lib):
    """Each ctypes declaration has the header's argument count, with a pointer
    exactly where the header has one and an int where it has an int or enum."""
    import ctypes
    text = open(os.path.join(ROOT, "include", "bsfa.h")).read()
    decls = re.findall(r"^(?:bsfa_status|const char\*)\s+(bsfa_\w+)\(([^;]*)\);", text, flags=re.M | re.S)
    assert sorted(n for n, _ in decls) == sorted(bsfa.EXPORTED)
    for name, args in decls:
        params = [a.strip() for a in args.replace("\n", " ").split(",") if a.strip() not in ("", "void")]
        want = [ctypes.c_void_p if "*" in a else ctypes.c_int for a in params]
        assert list(getattr(lib, name).argtypes) == want, name


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", bsfa.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (bsfa_\w+)", out))
    for name in _declared():
        assert name in exported, name
        assert hasattr(lib, name)


def test_status_strings(lib):
    assert bsfa.bsfa_status_string(0) == "BSFA_OK"
    assert bsfa.bsfa_status_string(4) == "BSFA_ERR_DEVICE_TIMEOUT"
    assert bsfa.bsfa_status_string(99) == "BSFA_UNKNOWN_STATUS"


@pytest.mark.parametrize("args,want", [
    ((1, 32, 8, 8192, 128, 128, 128, 1), bsfa.BSFA_OK),
    ((1, 2, 2, 512, 64, 64, 64, 1), bsfa.BSFA_OK),
    ((2, 24, 24, 16384, 128, 64, 128, 0), bsfa.BSFA_OK),
    ((0, 32, 8, 8192, 128, 128, 128, 1), bsfa.BSFA_ERR_INVALID_ARG),
    ((1, 32, 7, 8192, 128, 128, 128, 1), bsfa.BSFA_ERR_INVALID_ARG),
    ((1, -1, 1, 8192, 128, 128, 128, 1), bsfa.BSFA_ERR_INVALID_ARG),
    ((1, 32, 8, 8192, 96, 128, 128, 1), bsfa.BSFA_ERR_UNSUPPORTED),
    ((1, 32, 8, 8192, 128, 32, 128, 1), bsfa.BSFA_ERR_UNSUPPORTED),
    ((1, 32, 8, 8192, 128, 128, 256, 1), bsfa.BSFA_ERR_UNSUPPORTED),
    ((1, 32, 8, 8000, 128, 128, 128, 1), bsfa.BSFA_OK),          # ragged end
    ((1, 2, 2, 1, 64, 64, 128, 0), bsfa.BSFA_OK),               # a single token
    ((1, 8, 8, 4096 * 64 + 1, 64, 64, 64, 1), bsfa.BSFA_ERR_UNSUPPORTED),   # ceil(N/Bk) = 4097
    ((1024, 64, 8, 65536, 128, 128, 128, 1), bsfa.BSFA_ERR_UNSUPPORTED),
    ((1, 8, 8, 4096 * 64, 64, 64, 64, 1), bsfa.BSFA_OK),
    ((1, 8, 8, 4096 * 64 + 128, 64, 64, 64, 1), bsfa.BSFA_ERR_UNSUPPORTED),
])
def test_validate(lib, args, want):
    assert bsfa.bsfa_validate(*args) == want
    if want != bsfa.BSFA_OK:
        assert bsfa.bsfa_last_error()


def test_forward_rejects_bad_pointers_without_touching_cuda(lib):
    shape = (1, 2, 2, 512, 64, 64, 64, 1)
    # null q
    assert bsfa.bsfa_forward(None, 16, 16, 16, 16, None, None, *shape, None) == bsfa.BSFA_ERR_INVALID_ARG
    # misaligned k
    assert bsfa.bsfa_forward(16, 24, 16, 16, 16, None, None, *shape, None) == bsfa.BSFA_ERR_INVALID_ARG
    # misaligned lse
    assert bsfa.bsfa_forward(16, 16, 16, 16, 16, 2, None, *shape, None) == bsfa.BSFA_ERR_INVALID_ARG
    # unsupported shape wins before pointer checks
    assert bsfa.bsfa_forward(None, None, None, None, None, None, None, 1, 2, 2, 500, 96, 64, 64, 1, None) \
        == bsfa.BSFA_ERR_UNSUPPORTED


def test_tau_table_entry_rejects_bad_arguments_without_touching_cuda(lib):
    shape = (1, 2, 2, 500, 64, 64, 64, 1)
    for tiles in (0, -3):
        assert bsfa.bsfa_forward_tau_table(16, 16, 16, 16, tiles, 16, None, None, *shape, None) \
            == bsfa.BSFA_ERR_INVALID_ARG
        assert "tau_tiles" in bsfa.bsfa_last_error()
    assert bsfa.bsfa_forward_tau_table(16, 16, 16, None, 4, 16, None, None, *shape, None) == bsfa.BSFA_ERR_INVALID_ARG
    assert bsfa.bsfa_forward_tau_table(16, 16, 16, 18, 4, 16, None, None, *shape, None) == bsfa.BSFA_ERR_INVALID_ARG


def test_varlen_entry_rejects_bad_arguments_without_touching_cuda(lib):
    args = dict(total=1000, Hq=4, Hkv=2, D=128, Bq=128, Bk=128, causal=1)
    call = lambda cu, nseq, max_len, D=128: bsfa.bsfa_forward_varlen(16, 16, 16, cu, nseq, max_len, 16, 16, None, None,
                                                                      1000, 4, 2, D, 128, 128, 1, None)
    assert call(None, 2, 500) == bsfa.BSFA_ERR_INVALID_ARG          # no offsets
    assert call(16, 0, 500) == bsfa.BSFA_ERR_INVALID_ARG            # no sequences
    assert call(16, 2, 0) == bsfa.BSFA_ERR_INVALID_ARG              # no length
    assert call(18, 2, 500) == bsfa.BSFA_ERR_INVALID_ARG            # misaligned offsets
    assert call(16, 2, 4097 * 128) == bsfa.BSFA_ERR_UNSUPPORTED     # too many key blocks
    assert call(16, 2, 500, D=96) == bsfa.BSFA_ERR_UNSUPPORTED      # head dimension


def test_varlen_limit_is_per_sequence_not_per_batch(lib):
    """The 4096-key-block limit bounds each packed sequence (max_seqlen), not the
    packed total: a batch of many short sequences whose total exceeds 4096*Bk
    passes the shape checks. The misaligned out pointer then stops the call
    before any CUDA call, so the error names the alignment, not the size."""
    total = 4096 * 64 + 4097
    st = bsfa.bsfa_forward_varlen(16, 16, 16, 16, 300, 1000, 16, 0x1001, None, None, total, 2, 1, 64, 64, 64, 1, None)
    assert st == bsfa.BSFA_ERR_INVALID_ARG, bsfa.bsfa_last_error()
    assert "aligned" in bsfa.bsfa_last_error()
    # the same total is still refused for one sequence that long
    st = bsfa.bsfa_forward_varlen(16, 16, 16, 16, 1, total, 16, 0x1001, None, None, total, 2, 1, 64, 64, 64, 1, None)
    assert st == bsfa.BSFA_ERR_UNSUPPORTED and "key blocks" in bsfa.bsfa_last_error()
    # and a total whose rows overflow the 32-bit lse index
    st = bsfa.bsfa_forward_varlen(16, 16, 16, 16, 4, 1000, 16, 16, None, None, 2**30, 4, 1, 64, 64, 64, 1, None)
    assert st == bsfa.BSFA_ERR_UNSUPPORTED and "32-bit" in bsfa.bsfa_last_error()


def test_head_shard_entry_rejects_bad_ranges_without_touching_cuda(lib):
    call = lambda b, c: bsfa.bsfa_forward_heads(16, 16, 16, 16, 16, None, None, 1, 8, 4, 512, 128, 128, 128, 1, b, c,
                                                None)
    for b, c in ((-1, 2), (0, 0), (0, -1), (3, 2), (4, 1)):
        assert call(b, c) == bsfa.BSFA_ERR_INVALID_ARG, (b, c)
        assert "kv" in bsfa.bsfa_last_error().lower() or "heads" in bsfa.bsfa_last_error()


def test_row_range_entry_rejects_bad_ranges_without_touching_cuda(lib):
    call = lambda b, e: bsfa.bsfa_forward_rows(16, 16, 16, 16, 16, None, None, 1, 8, 4, 1000, 128, 128, 128, 1, b, e,
                                               None)
    for b, e in ((-256, 256), (128, 512), (256, 256), (512, 256), (0, 1001), (0, -1), (1024, 1000)):
        assert call(b, e) == bsfa.BSFA_ERR_INVALID_ARG, (b, e)
        assert "row" in bsfa.bsfa_last_error(), bsfa.bsfa_last_error()


def test_host_buffer_entry_rejects_bad_arguments_without_touching_cuda(lib):
    ptrs = [16] * 12
    shape = (1, 8, 4, 512, 128, 128, 128, 1)
    assert bsfa.bsfa_forward_host(*ptrs, *shape, 0, None) == bsfa.BSFA_ERR_INVALID_ARG        # no chunks
    assert bsfa.bsfa_forward_host(*ptrs, *shape, 3, None) == bsfa.BSFA_ERR_INVALID_ARG        # more chunks than
    assert "256" in bsfa.bsfa_last_error()                                                     # 256-row units
    missing = list(ptrs)
    missing[6] = None                                                                          # no device q
    assert bsfa.bsfa_forward_host(*missing, *shape, 2, None) == bsfa.BSFA_ERR_INVALID_ARG
    half_lse = list(ptrs)
    half_lse[11] = None                                                                        # lse on one side only
    assert bsfa.bsfa_forward_host(*half_lse, *shape, 2, None) == bsfa.BSFA_ERR_INVALID_ARG
    assert bsfa.bsfa_forward_host(*ptrs, 1, 8, 4, 512, 96, 128, 128, 1, 2, None) == bsfa.BSFA_ERR_UNSUPPORTED


def test_host_buffer_binding_checks_layouts_before_any_copy():
    """forward_host hands raw host addresses and device buffers to the C call, so
    wrong dtypes, strides or buffer shapes must be refused before it runs."""
    import torch
    B, N, Hq, Hkv, D = 1, 96, 4, 2, 64
    q = torch.zeros((B, N, Hq, D), dtype=torch.bfloat16)
    k = torch.zeros((B, N, Hkv, D), dtype=torch.bfloat16)
    v = torch.zeros_like(k)
    tau = torch.zeros(Hq, dtype=torch.float32)
    bufs = {"q": q.clone(), "k": k.clone(), "v": v.clone(), "tau": tau.clone(), "out": q.clone(),
            "lse": torch.zeros((B, Hq, N)), "out_host": q.clone(), "lse_host": torch.zeros((B, Hq, N))}
    bsfa._check_host_inputs(q, k, v, tau, bufs)               # consistent: accepted
    bsfa._check_host_inputs(q, k, v, tau, None)

    call = lambda *a, b=bufs: bsfa.forward_host(*a, Bq=64, Bk=64, causal=True, bufs=b)
    bad_inputs = [
        (q.float(), k, v, tau),                                # wrong dtype
        (q.transpose(1, 2), k, v, tau),                        # not contiguous
        (q, k[:, :48], v, tau),                                # k shorter than q
        (q, k, v[..., :32].contiguous(), tau),                 # v's head dimension
        (q, k, v, tau[:3]),                                    # one threshold short
        (q, k, v, tau.double()),                               # wrong threshold dtype
    ]
    for args in bad_inputs:
        with pytest.raises(ValueError):
            call(*args)
    for name, bad in (("out", torch.zeros((B, N - 1, Hq, D), dtype=torch.bfloat16)),
                      ("k", torch.zeros((B, N, Hq, D), dtype=torch.bfloat16)),
                      ("lse_host", torch.zeros((B, Hq, N), dtype=torch.bfloat16)),
                      ("tau", None)):
        b = dict(bufs)
        b[name] = bad
        with pytest.raises(ValueError):
            call(q, k, v, tau, b=b)
