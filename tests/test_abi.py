"""The C ABI: the library loads, exports every function include/fa.h declares, and its
host-side validation rejects bad arguments before touching a device (runs without a
GPU: no call here reaches a kernel)."""
import ctypes
import os
import re

import pytest

from exact_io_aware_64_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    inc = os.path.join(ROOT, "include")
    for fn in os.listdir(inc):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(inc, fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b(fa_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    return binding.lib()


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("fa_fwd", "fa_bwd", "fa_fwd_f32", "fa_bwd_f32",
                     "fa_bwd_workspace_bytes", "fa_status_string", "fa_check_device_error"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name
    # the binding's signature table covers the same set
    assert set(binding.SIGNATURES) == set(_declared_functions())


def test_status_strings(lib):
    assert binding.status_name(0) == "FA_OK"
    assert binding.status_name(1) == "FA_ERR_INVALID_ARG"
    assert binding.status_name(2) == "FA_ERR_UNSUPPORTED"
    assert binding.status_name(3) == "FA_ERR_CUDA"
    assert binding.status_name(4) == "FA_ERR_TIMEOUT"
    assert lib.fa_abi_version() == 1


def test_workspace_is_linear_in_rows(lib):
    # two float32 per row (D and LSE*log2e), rows padded to whole 128-row tiles
    assert binding.workspace_bytes(2, 16, 8192, 128) == 2 * 2 * 16 * 8192 * 4
    assert binding.workspace_bytes(1, 1, 1, 64) == 2 * 128 * 4
    assert binding.workspace_bytes(1, 32, 10000, 128) == 2 * 32 * 10112 * 4
    assert binding.workspace_bytes(0, 4, 128, 64) == 0
    # O(B*H*N), never O(N^2): the backward stores no score tile
    assert binding.workspace_bytes(1, 1, 32768, 128) == 2 * 32768 * 4


# Fake, 16-byte aligned addresses: validation must fail (or finish) before any use.
A, B_, C, D_, E = 0x100000, 0x200000, 0x300000, 0x400000, 0x500000


def _fwd(lib, q=A, k=B_, v=C, o=D_, lse=E, B=1, H=1, N=16, d=64, scale=0.125, causal=0):
    st = lib.fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, None)
    return st, lib.fa_last_error_message().decode()


def test_fwd_validation(lib):
    assert _fwd(lib, q=0)[0] == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, o=0)[0] == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, k=B_ + 8)[0] == binding.FA_ERR_INVALID_ARG      # misaligned
    assert _fwd(lib, d=96)[0] == binding.FA_ERR_UNSUPPORTED
    assert _fwd(lib, d=256)[0] == binding.FA_ERR_UNSUPPORTED
    assert _fwd(lib, N=-1)[0] == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, scale=0.0)[0] == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, scale=float("nan"))[0] == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, scale=float("inf"))[0] == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, causal=2)[0] == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, o=A + 16)[0] == binding.FA_ERR_INVALID_ARG       # O overlaps Q
    assert _fwd(lib, lse=E + 2)[0] == binding.FA_ERR_INVALID_ARG      # LSE misaligned
    st, msg = _fwd(lib, d=96)
    assert "d=96" in msg
    huge = _fwd(lib, B=1 << 15, H=1 << 15, N=1 << 12)
    assert huge[0] == binding.FA_ERR_INVALID_ARG
    # lengths near INT_MAX: rounded up to whole 256-row units they would overflow a
    # 32-bit int, so they are rejected before any arithmetic on them
    for n in ((1 << 31) - 1, (1 << 31) - 255):
        st, msg = _fwd(lib, N=n)
        assert st == binding.FA_ERR_INVALID_ARG and "too large" in msg, msg
    assert lib.fa_fwd_qk(A, B_, C, D_, E, 1, 1, 16, (1 << 31) - 1, 64, 0.1, 0,
                         None) == binding.FA_ERR_INVALID_ARG
    # the workspace size of such a length is computed without overflow
    n = (1 << 31) - 1
    assert binding.workspace_bytes(1, 1, n, 64) == 2 * ((n + 127) // 128 * 128) * 4


def test_empty_problems_are_noops(lib):
    # N = 0 or B*H = 0: nothing to do, no device needed
    assert _fwd(lib, N=0)[0] == binding.FA_OK
    assert _fwd(lib, B=0)[0] == binding.FA_OK
    assert lib.fa_fwd_f32(A, B_, C, D_, E, 1, 3, 0, 128, 0.1, 1, None) == binding.FA_OK


@pytest.mark.parametrize("fn,elem", [("fa_bwd", 2), ("fa_bwd_f32", 4)])
def test_bwd_validation(lib, fn, elem):
    F, G, H_, I, J = 0x600000, 0x700000, 0x800000, 0x900000, 0xA00000
    args = [A, B_, C, D_, E, F, G, H_, I, 1, 2, 64, 128, 0.1, 1, J, 1 << 20, None]
    call_fn = getattr(lib, fn)

    def call(**kw):
        a = list(args)
        names = ["Q", "K", "V", "O", "dO", "LSE", "dQ", "dK", "dV", "B", "H", "N", "d",
                 "scale", "causal", "ws", "ws_bytes", "stream"]
        for k, v in kw.items():
            a[names.index(k)] = v
        return call_fn(*a)

    assert call(B=0) == binding.FA_OK                      # empty: no-op
    assert call(N=0, Q=0, dQ=0) == binding.FA_OK           # empty: NULL pointers allowed
    assert lib.fa_fwd(0, 0, 0, 0, 0, 1, 1, 0, 64, 0.1, 0, None) == binding.FA_OK
    assert call(LSE=0) == binding.FA_ERR_INVALID_ARG        # LSE required
    assert call(dO=0) == binding.FA_ERR_INVALID_ARG
    assert call(ws=0) == binding.FA_ERR_INVALID_ARG
    assert call(ws_bytes=100) == binding.FA_ERR_INVALID_ARG
    assert call(d=80) == binding.FA_ERR_UNSUPPORTED
    assert call(causal=3) == binding.FA_ERR_INVALID_ARG
    assert call(scale=-1.0) == binding.FA_ERR_INVALID_ARG
    assert call(dQ=A) == binding.FA_ERR_INVALID_ARG         # gradient overlaps an input
    assert call(dK=G) == binding.FA_ERR_INVALID_ARG         # gradients overlap
    assert call(ws=H_) == binding.FA_ERR_INVALID_ARG        # workspace overlaps dK
    # the overlap checks use the element size: a gradient that ends where the next
    # buffer starts does not overlap it, one element more does
    row = 1 * 1 * 1 * 64 * elem
    small = [A, B_, C, D_, E, F, G, H_, I, 1, 1, 1, 64, 0.1, 0, I + row, 1024, None]
    assert call_fn(*small) != binding.FA_ERR_INVALID_ARG
    small[15] = I + row - 16
    assert call_fn(*small) == binding.FA_ERR_INVALID_ARG


def test_trace_events_validation(lib):
    assert lib.fa_trace_events(None, 0) == binding.FA_OK
    assert lib.fa_trace_events(None, 2) == binding.FA_ERR_INVALID_ARG
    assert lib.fa_trace_events(None, -1) == binding.FA_ERR_INVALID_ARG
    arr = (ctypes.c_void_p * 9)()
    assert lib.fa_trace_events(arr, 9) == binding.FA_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        binding.lib()


def test_qk_validation(lib):
    """fa_fwd_qk / fa_bwd_qk: Nq queries against Nk keys (queries = the last Nq tokens)."""
    def fwd(Nq, Nk, causal=1, o=D_, **kw):
        return lib.fa_fwd_qk(A, B_, C, o, E, 1, 2, Nq, Nk, 64, 0.1, causal, None)

    assert fwd(0, 5) == binding.FA_OK                      # no queries: no-op
    assert fwd(4, 0) == binding.FA_ERR_INVALID_ARG         # queries without keys
    assert fwd(8, 4, causal=1) == binding.FA_ERR_INVALID_ARG  # causal needs Nq <= Nk
    assert "Nq <= Nk" in lib.fa_last_error_message().decode()
    assert fwd(8, 4, causal=0) != binding.FA_ERR_INVALID_ARG  # non-causal: any lengths
    assert fwd(-1, 4) == binding.FA_ERR_INVALID_ARG
    # O is sized by Nq, K and V by Nk: O right after a short K does not overlap it
    assert fwd(16, 64, o=B_ + 2 * 64 * 64 * 2) != binding.FA_ERR_INVALID_ARG
    assert fwd(16, 64, o=B_ + 2 * 64 * 64 * 2 - 16) == binding.FA_ERR_INVALID_ARG

    F, G, H_, I, J = 0x600000, 0x700000, 0x800000, 0x900000, 0xA00000

    def bwd(Nq, Nk, causal=1, ws_bytes=1 << 20, dk=H_):
        return lib.fa_bwd_qk(A, B_, C, D_, E, F, G, dk, I, 1, 2, Nq, Nk, 64, 0.1, causal, J,
                             ws_bytes, None)

    assert bwd(0, 0) == binding.FA_OK
    # keys without queries: dK and dV get zeros, so they are checked before the device is
    assert bwd(0, 3, dk=0) == binding.FA_ERR_INVALID_ARG
    assert "dK" in lib.fa_last_error_message().decode()
    assert bwd(0, 3, dk=H_ + 8) == binding.FA_ERR_INVALID_ARG
    assert bwd(5, 3) == binding.FA_ERR_INVALID_ARG
    assert bwd(3, 0) == binding.FA_ERR_INVALID_ARG
    # the workspace is sized by the query rows
    need = binding.workspace_bytes(1, 2, 100, 64)
    assert bwd(100, 1000, ws_bytes=need - 4) == binding.FA_ERR_INVALID_ARG
    assert bwd(100, 1000, ws_bytes=need) != binding.FA_ERR_INVALID_ARG
    assert bwd(100, 1000, dk=G + 2 * 100 * 64 * 2 - 16) == binding.FA_ERR_INVALID_ARG


def test_varlen_validation(lib):
    """fa_fwd_varlen / fa_bwd_varlen: the length arrays are required (values are checked on
    the device); the padded shapes follow the fa_fwd_qk rules."""
    SQ, SK = 0xB00000, 0xC00000
    def fwd(sq=SQ, sk=SK, Nq=64, Nk=64, causal=1):
        return lib.fa_fwd_varlen(A, B_, C, D_, E, sq, sk, 2, 2, Nq, Nk, 64, 0.1, causal, None)

    assert fwd(sq=0) == binding.FA_ERR_INVALID_ARG
    assert fwd(sk=0) == binding.FA_ERR_INVALID_ARG
    assert fwd(sq=SQ + 2) == binding.FA_ERR_INVALID_ARG      # misaligned
    assert fwd(Nq=128, Nk=64) == binding.FA_ERR_INVALID_ARG   # causal: padded Nq <= Nk
    assert fwd(Nq=0, sq=0, sk=0) == binding.FA_OK             # empty: no-op
    F, G, H_, I, J = 0x600000, 0x700000, 0x800000, 0x900000, 0xA00000
    st = lib.fa_bwd_varlen(A, B_, C, D_, E, F, G, H_, I, 0, SK, 2, 2, 64, 64, 64, 0.1, 1, J,
                           1 << 20, None)
    assert st == binding.FA_ERR_INVALID_ARG


def test_merge_validation(lib):
    O_acc, L_acc, O_p, L_p, O_out = 0x100000, 0x200000, 0x300000, 0x400000, 0x500000

    def call(oa=O_acc, la=L_acc, op=O_p, lp=L_p, oo=O_out, N=16, d=64):
        return lib.fa_merge(oa, la, op, lp, oo, 1, 2, N, d, None)

    assert call(N=0, oa=0, la=0, op=0, lp=0) == binding.FA_OK   # empty: no-op
    assert call(la=0) == binding.FA_ERR_INVALID_ARG
    assert call(op=0) == binding.FA_ERR_INVALID_ARG
    assert call(oa=O_acc + 8) == binding.FA_ERR_INVALID_ARG    # misaligned
    assert call(lp=L_p + 2) == binding.FA_ERR_INVALID_ARG
    assert call(d=96) == binding.FA_ERR_UNSUPPORTED
    assert call(op=O_acc + 64) == binding.FA_ERR_INVALID_ARG   # accumulator overlaps part
    assert call(oo=O_acc) == binding.FA_ERR_INVALID_ARG        # output overlaps accumulator
    assert call(oo=0) != binding.FA_ERR_INVALID_ARG            # no bf16 output is fine


def test_accumulate_validation(lib):
    acc, part, out = 0x100000, 0x200000, 0x300000
    assert lib.fa_accumulate(0, 0, 0, 0, None) == binding.FA_OK          # n = 0: no-op
    assert lib.fa_accumulate(acc, part, out, 12, None) == binding.FA_ERR_INVALID_ARG  # not /8
    assert lib.fa_accumulate(0, part, out, 16, None) == binding.FA_ERR_INVALID_ARG
    assert lib.fa_accumulate(acc + 4, part, out, 16, None) == binding.FA_ERR_INVALID_ARG
    assert lib.fa_accumulate(acc, acc + 32, 0, 16, None) == binding.FA_ERR_INVALID_ARG  # overlap
    assert lib.fa_accumulate(acc, part, acc + 16, 16, None) == binding.FA_ERR_INVALID_ARG


def test_selftest_timeout_validation(lib):
    assert lib.fa_selftest_timeout(-1, None) == binding.FA_ERR_INVALID_ARG
    assert lib.fa_selftest_timeout(1 << 35, None) == binding.FA_ERR_INVALID_ARG


def test_packed_validation(lib):
    CQ, CK = 0xB00000, 0xC00000

    def fwd(cq=CQ, ck=CK, maxq=64, maxk=64, tq=100, tk=100, causal=1):
        return lib.fa_fwd_packed(A, B_, C, D_, E, cq, ck, 2, 2, maxq, maxk, tq, tk, 64, 0.1,
                                 causal, None)

    assert fwd(tq=0, cq=0, ck=0) == binding.FA_OK             # no tokens: no-op
    assert fwd(cq=0) == binding.FA_ERR_INVALID_ARG
    assert fwd(ck=CK + 2) == binding.FA_ERR_INVALID_ARG       # misaligned
    assert fwd(maxq=128, maxk=64) == binding.FA_ERR_INVALID_ARG  # causal: max_q <= max_k
    assert fwd(tq=-1) == binding.FA_ERR_INVALID_ARG
    F, G, H_, I, J = 0x600000, 0x700000, 0x800000, 0x900000, 0xA00000
    need = binding.workspace_bytes(2, 2, 64, 64)
    st = lib.fa_bwd_packed(A, B_, C, D_, E, F, G, H_, I, CQ, CK, 2, 2, 64, 64, 100, 100, 64,
                           0.1, 1, J, need - 4, None)
    assert st == binding.FA_ERR_INVALID_ARG                   # workspace too small


def test_binding_refuses_host_tensors():
    """No CPU fallback: every entry point of the binding rejects tensors that are not on a
    CUDA device before anything is computed."""
    import torch
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    lse = torch.zeros(1, 1, 8)
    with pytest.raises(ValueError, match="CUDA"):
        binding.fwd(q, q, q)
    with pytest.raises(ValueError, match="CUDA"):
        binding.bwd(q, q, q, q, q, lse)
    with pytest.raises(ValueError, match="CUDA"):
        binding.bwd_noalloc(q, q, q, q, q, lse)
    with pytest.raises(ValueError, match="CUDA"):
        binding.fwd_packed(q[0, 0].unsqueeze(1), q[0, 0].unsqueeze(1), q[0, 0].unsqueeze(1),
                           torch.zeros(2, dtype=torch.int32), torch.zeros(2, dtype=torch.int32),
                           8, 8)
    with pytest.raises(ValueError):
        binding.merge(torch.zeros(1, 1, 8, 64), lse, q, lse)
    with pytest.raises(ValueError):
        binding.accumulate(torch.zeros(8), torch.zeros(8, dtype=torch.bfloat16))


def test_f32_layout_validation(lib):
    """The float32 Nq != Nk, padded and packed calls follow the bf16 rules, with 4-byte
    elements in the size and overlap checks."""
    F, G, H_, I, J = 0x600000, 0x700000, 0x800000, 0x900000, 0xA00000
    SQ, SK = 0xB00000, 0xC00000

    def fwd_qk(Nq, Nk, causal=1, o=D_):
        return lib.fa_fwd_f32_qk(A, B_, C, o, E, 1, 2, Nq, Nk, 64, 0.1, causal, None)

    assert fwd_qk(0, 5) == binding.FA_OK
    assert fwd_qk(4, 0) == binding.FA_ERR_INVALID_ARG
    assert fwd_qk(8, 4, causal=1) == binding.FA_ERR_INVALID_ARG
    assert fwd_qk(8, 4, causal=0) != binding.FA_ERR_INVALID_ARG
    # K holds 2 heads x 64 rows x 64 float32: O just past it does not overlap, 16 B less does
    assert fwd_qk(16, 64, o=B_ + 2 * 64 * 64 * 4) != binding.FA_ERR_INVALID_ARG
    assert fwd_qk(16, 64, o=B_ + 2 * 64 * 64 * 4 - 16) == binding.FA_ERR_INVALID_ARG

    def bwd_qk(Nq, Nk, ws_bytes=1 << 20, dk=H_):
        return lib.fa_bwd_f32_qk(A, B_, C, D_, E, F, G, dk, I, 1, 2, Nq, Nk, 64, 0.1, 1, J,
                                 ws_bytes, None)

    assert bwd_qk(5, 3) == binding.FA_ERR_INVALID_ARG
    need = binding.workspace_bytes(1, 2, 100, 64)
    assert bwd_qk(100, 1000, ws_bytes=need - 4) == binding.FA_ERR_INVALID_ARG
    assert bwd_qk(100, 1000, ws_bytes=need) != binding.FA_ERR_INVALID_ARG
    assert bwd_qk(100, 1000, dk=G + 2 * 100 * 64 * 4 - 16) == binding.FA_ERR_INVALID_ARG

    assert lib.fa_fwd_f32_varlen(A, B_, C, D_, E, 0, SK, 2, 2, 64, 64, 64, 0.1, 1,
                                 None) == binding.FA_ERR_INVALID_ARG
    assert lib.fa_fwd_f32_varlen(A, B_, C, D_, E, SQ, SK, 2, 2, 128, 64, 64, 0.1, 1,
                                 None) == binding.FA_ERR_INVALID_ARG
    assert lib.fa_bwd_f32_varlen(A, B_, C, D_, E, F, G, H_, I, SQ, 0, 2, 2, 64, 64, 64, 0.1,
                                 1, J, 1 << 20, None) == binding.FA_ERR_INVALID_ARG

    def fwd_packed(cq=SQ, ck=SK, tq=100, tk=100, o=D_):
        return lib.fa_fwd_f32_packed(A, B_, C, o, E, cq, ck, 2, 2, 64, 64, tq, tk, 64, 0.1, 1,
                                     None)

    assert fwd_packed(tq=0, cq=0, ck=0) == binding.FA_OK
    assert fwd_packed(cq=0) == binding.FA_ERR_INVALID_ARG
    # Q holds 100 tokens x 2 heads x 64 float32
    assert fwd_packed(o=A + 100 * 2 * 64 * 4 - 16) == binding.FA_ERR_INVALID_ARG
    need = binding.workspace_bytes(2, 2, 64, 64)
    st = lib.fa_bwd_f32_packed(A, B_, C, D_, E, F, G, H_, I, SQ, SK, 2, 2, 64, 64, 100, 100,
                               64, 0.1, 1, J, need - 4, None)
    assert st == binding.FA_ERR_INVALID_ARG
